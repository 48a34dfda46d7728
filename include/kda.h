/*
 * kda.h -- C ABI of a B200 (sm_100a) implementation of Kimi Delta Attention.
 *
 * KDA is a gated delta-rule linear attention with one forget gate per key
 * channel ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
 * Background: Gated DeltaNet's scalar gate widened to a diagonal matrix).
 * For one (sequence, head), with a D_k x D_v FP32 state S (row = key channel):
 *
 *     alpha_t = exp(g_t)                           (natural log-decay, per channel)
 *     S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t     = S_t^T q_t
 *
 * Preconditions on the data (not checked on the device): g in [-5, 0] (the
 * lower-bounded decay of "MoonshotAI/Kimi-K3 딥다이브" (fiv.co.kr/repos/kimi-k3-deep-dive.html),
 * section 4-1),
 * beta in [0, 1], finite inputs.  No 1/sqrt(D) scale is applied to q, and q,
 * k, beta, g are used as given (no normalisation, sigmoid or clamp inside).
 *
 * Layouts (all dense, row-major, no padding):
 *   q, k, g : [T_tot, H, D_k]     v, out : [T_tot, H, D_v]     beta : [T_tot, H]
 *   states  : [N, H, D_k, D_v] FP32
 *   checkpoints : [n_ckpt, H, D_k, D_v] FP32, packed sequence by sequence.
 * q, k, v and out share one dtype (FP32 or BF16); g, beta and states are FP32.
 *
 * Ownership and streams: the caller owns every buffer it passes; all
 * pointers are device pointers unless a comment says "host".  Every call is
 * asynchronous on the given stream and never synchronises.  The library
 * itself holds device memory in exactly two places:
 *   - kda_prefill's workspace pool: on the first kda_prefill call on a device
 *     the library creates a CUDA memory pool for that device.  Each call on
 *     the two-pass path (kda_prefill_path = 2) takes one workspace from it,
 *     at most the pool cap (8 GiB unless kda_set_workspace_pool_cap says
 *     otherwise; longer inputs run in windows of chunks), and gives it back
 *     at the end of the call, ordered on the call's stream.  The pool keeps
 *     what it has been given back (release threshold: unlimited), so later
 *     calls reuse the memory without allocating; kda_release_workspace_pool
 *     returns it to the device.  When even the smallest window does not fit
 *     under the cap, or the pool cannot supply it, the call runs the
 *     single-pass tensor-core kernel instead (same results within the
 *     tolerances, about 20 % slower); kda_last_prefill_path tells which ran.
 *   - the fixed array of KDA_NOALLOC_SCRATCH_BYTES behind
 *     kda_prefill_noalloc, present on every device that loads the library.
 * kda_prefill_ws, kda_prefill_at, the decode and backward calls and the
 * affine maps take no device memory of their own.
 *
 * Errors: argument problems return KDA_ERR_INVALID_ARGUMENT or
 * KDA_ERR_UNSUPPORTED before anything is launched.  A failed launch returns
 * KDA_ERR_CUDA; kda_last_cuda_error() gives the cudaError_t value.  Kernels
 * with bounded waits write KDA_ERR_TIMEOUT to shape->dev_status (when it is
 * not NULL) instead of hanging; the caller reads it after synchronising.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misalignment          */
  KDA_ERR_UNSUPPORTED = 2,      /* a head size or chunk size the library lacks   */
  KDA_ERR_CUDA = 3,             /* a CUDA call failed; see kda_last_cuda_error() */
  KDA_ERR_TIMEOUT = 4           /* written to dev_status by a bounded wait       */
} kda_status;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype;

typedef struct {
  int32_t num_seqs;     /* N >= 1                                                  */
  int64_t total_tokens; /* T_tot = cu_seqlens[N] (prefill); N (decode)             */
  int32_t num_heads;    /* H >= 1                                                  */
  int32_t head_dim_k;   /* D_k in {32, 64, 128}                                    */
  int32_t head_dim_v;   /* D_v in {32, 64, 128}                                    */
  int32_t chunk;        /* C in {16, 64} (prefill); ignored by decode              */
  int32_t qkv_dtype;    /* kda_dtype of q, k, v and out                            */
  int32_t *dev_status;  /* optional device int32, 0 = fine, else a kda_status      */
} kda_shape;

/*
 * Chunked prefill ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
 * Methods 1, FlashKDA: the recurrence unrolled over chunks into matrix
 * products; "MoonshotAI/Kimi-K3 딥다이브" (fiv.co.kr/repos/kimi-k3-deep-dive.html),
 * section 4-1: 16-token tiles with a recurrence between tiles) and state
 * checkpoints for prefix caching ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557), Methods 3: the state is kept only
 * at coarse positions such as every 32K tokens).
 *
 *   q, k, v, g, beta : inputs in the layouts above (beta needs 4-byte alignment).
 *   init_state       : [N, H, D_k, D_v] or NULL for zeros (append-prefill
 *                      after a cached prefix passes the cached state here).
 *   cu_seqlens       : device int32[N+1], cu_seqlens[0] = 0, non-decreasing,
 *                      cu_seqlens[N] = total_tokens.  Not checked on the device.
 *   out              : [T_tot, H, D_v], written for every token.
 *   final_state      : [N, H, D_k, D_v] or NULL; may alias init_state.
 *   ckpt_interval    : 0 = no checkpoints; else a positive multiple of chunk.
 *                      Sequence i stores its state after every ckpt_interval
 *                      of its own tokens (counted from its first token, the
 *                      end included when T_i is a multiple).
 *   ckpt_states      : [kda_ckpt_count(...), H, D_k, D_v]; NULL iff interval 0.
 * Every other pointer must be 16-byte aligned; out must not overlap any input.
 *
 * Kernels: BF16 with D_k = D_v = 128 runs on the tensor cores (tcgen05) for
 * chunk 16 and chunk 64 alike.  The tensor-core kernels group tokens in
 * chunks of 64 with 16-token diagonal blocks inside; the result does not
 * depend on the chunk size, which the caller names only to fix which
 * checkpoint intervals are valid.  With up to 1024 sequences and 2048
 * (sequence, head) units and an interval that is 0 or a multiple of 64 the
 * call runs the two-pass kernels through the workspace pool, unless the
 * windows that workspace allows would cost more than the work (see
 * kda_prefill_path); larger batches, or an interval of 16, 32 or 48 modulo
 * 64, run the single-pass tensor-core kernel.  Other shapes (FP32, smaller
 * heads) run the FP32 SIMT kernel.
 */
kda_status kda_prefill(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *init_state, const int32_t *cu_seqlens,
                       void *out, float *final_state, int64_t ckpt_interval,
                       float *ckpt_states, const kda_shape *shape, kda_stream_t stream);

/*
 * kda_prefill with a caller-owned device workspace.  Shapes on the two-pass
 * tensor-core path (kda_prefill_path = 2) store one packet of intra-chunk
 * products per (chunk, head) in the workspace, then run the inter-chunk
 * chain over them.  workspace_bytes >= kda_prefill_workspace_bytes(shape)
 * runs the whole batch in one window; a smaller workspace (at least
 * kda_prefill_workspace_min_bytes) runs it in several windows of chunks.
 * A NULL or too small workspace, a shape off the two-pass path, or windows
 * that would cost more than the work (see kda_prefill_path) run the
 * single-pass kernels, which need none.  The workspace must be 16-byte
 * aligned (256 is best), must not overlap any argument, and is free again
 * when the work queued on `stream` completes.  kda_prefill itself takes its
 * workspace from a memory pool the library keeps per device (released by
 * kda_release_workspace_pool).
 */
kda_status kda_prefill_ws(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *init_state, const int32_t *cu_seqlens,
                          void *out, float *final_state, int64_t ckpt_interval,
                          float *ckpt_states, void *workspace, size_t workspace_bytes,
                          const kda_shape *shape, kda_stream_t stream);

/* Size of the fixed device array behind kda_prefill_noalloc. */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20)

/*
 * kda_prefill for callers that cannot allocate device memory when they call
 * it: a serving engine that has already handed all free memory to its own
 * pool (a KV cache sized to what was left), or a runtime whose allocator this
 * library cannot reach.  It runs the two-pass prefill with its workspace in
 * a fixed array of KDA_NOALLOC_SCRATCH_BYTES compiled into the library (every
 * GPU that loads the library holds it until the process exits) and calls no
 * allocator.  No part of the methods on the pages this library follows
 * corresponds to it; it is a deployment aid.
 *
 * Arguments as for kda_prefill.  Only shapes on the two-pass path
 * (kda_prefill_path = 2) are accepted, and only when one chunk of every
 * (sequence, head) fits the array: num_seqs * num_heads * 74240 bytes, plus
 * num_seqs * num_heads * 65536 when final_state is NULL, plus 256, at most
 * KDA_NOALLOC_SCRATCH_BYTES; longer batches run in windows of chunks, or on
 * the single-pass kernel (which needs no workspace) where those windows would
 * cost more than the work, as in kda_prefill_ws.  Other shapes return
 * KDA_ERR_UNSUPPORTED before any work is queued.
 * The first call on a device looks up the array's device address, so make
 * that first call before any stream capture.  The address is kept for the
 * life of the process: after cudaDeviceReset (or anything else that tears
 * down and recreates the device's primary context) this entry point must not
 * be called again in that process.  All calls share the one array
 * and nothing in it needs to start at zero (each call writes every byte it
 * reads), but calls whose work overlaps on the GPU (other streams, other
 * threads) race on it: order them on one stream or synchronise between them.
 */
kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *init_state,
                               const int32_t *cu_seqlens, void *out, float *final_state,
                               int64_t ckpt_interval, float *ckpt_states,
                               const kda_shape *shape, kda_stream_t stream);

/*
 * kda_prefill with states also stored at explicit positions, such as the
 * boundaries of cached prompts (the first page, Conclusion table: prefix
 * caching keeps the state every 32K tokens "+ prompt boundaries").
 *
 *   pos_cu     : device int32[N+1], offsets into positions (pos_cu[0] = 0).
 *   positions  : device int32; entries pos_cu[i] .. pos_cu[i+1]-1 are token
 *                counts of sequence i, in increasing order.
 *   pos_states : [pos_cu[N], H, D_k, D_v] FP32; entry j receives the state
 *                after positions[j] tokens of its sequence.
 * An entry <= 0 stores the initial state, an entry >= T_i the final state,
 * and an entry not larger than its predecessor the same state as it.  The
 * three pointers are all NULL (no positions; this is kda_prefill) or all
 * set.  Chunks are cut at every position, so the result does not depend on
 * where the positions fall; each position that is not a multiple of the
 * chunk adds one partial chunk.  Other arguments as for kda_prefill.
 */
kda_status kda_prefill_at(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *init_state, const int32_t *cu_seqlens,
                          void *out, float *final_state, int64_t ckpt_interval,
                          float *ckpt_states, const int32_t *pos_cu, const int32_t *positions,
                          float *pos_states, const kda_shape *shape, kda_stream_t stream);

/*
 * One decode step for N sequences ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
 * Methods 1: decode runs the
 * recurrence directly; about 7 D^2 FLOPs and 8 D^2 bytes of FP32 state
 * traffic per head per token).
 *
 *   q, k, v, g : [N, H, D]   beta : [N, H]   out : [N, H, D_v]
 *   state_inout: [N, H, D_k, D_v], read and overwritten in place.
 * shape->total_tokens must equal shape->num_seqs; shape->chunk is ignored.
 */
kda_status kda_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state_inout, void *out,
                      const kda_shape *shape, kda_stream_t stream);

/*
 * Multi-token decode for speculative-decoding verification: every sequence
 * brings tokens_per_seq new tokens (a draft), all of them run through the
 * recurrence from state_inout, the output of every token is written, and
 * state_inout is then replaced by the state reached after the first
 * accept_len[n] tokens of sequence n (0 leaves it unchanged).  accept_len
 * may be NULL: all tokens are accepted.  The state crosses HBM once per call.
 *
 *   q, k, g : [N, tokens_per_seq, H, D_k]   v, out : [N, tokens_per_seq, H, D_v]
 *   beta    : [N, tokens_per_seq, H]         accept_len : device int32[N] or NULL
 *   state_inout : [N, H, D_k, D_v]
 * shape->total_tokens must equal N * tokens_per_seq; 1 <= tokens_per_seq <= 64.
 * Values of accept_len outside [0, tokens_per_seq] are clamped.  The result
 * is the recurrence of the decode step applied token by token (the first
 * page, Methods 1: decode runs the recurrence directly).  BF16 inputs with
 * D_k = D_v = 128 and at most 16 tokens compute it as one chunk of the
 * chunked form (Methods 1, FlashKDA) on the tensor cores, with S0 rounded to
 * BF16 as an operand and the state updated in FP32; other shapes run the
 * recurrence on the CUDA cores.  The serving side that decides acceptance is
 * not part of this library.
 */
kda_status kda_decode_multi(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *state_inout, void *out,
                            const int32_t *accept_len, int32_t tokens_per_seq,
                            const kda_shape *shape, kda_stream_t stream);

/*
 * Backward pass of the recurrence, for training (the pages name training work
 * but give no detail; the gradients follow from the forward definition above
 * by reverse-mode differentiation).
 *
 * BF16 q/k/v with D_k = D_v = 128 and at most 1024 sequences run the chunked
 * form on the tensor cores when the workspace is at least
 * kda_backward_workspace_bytes(shape) (what that query returns for such
 * shapes): the forward is recomputed by the two-pass prefill (its intra-chunk
 * packets and, every 64 tokens, the state as a BF16 tile kept in the
 * workspace), then a chain kernel carries the state gradient backwards chunk
 * by chunk and two kernels, one after the other and each over all (chunk,
 * head) items at once, form every chunk's gradients from 64 x 64 and
 * 64 x 128 tcgen05 products.  The workspace then holds about 250 KB per
 * (64-token chunk, head).
 * Other shapes, or a smaller workspace that still covers the SIMT kernel's
 * need, run the FP32 SIMT kernel token by token; kda_last_backward_path tells
 * which ran.
 *
 *   q, k, v, g, beta, init_state, cu_seqlens : the forward call's inputs
 *   d_out         : [T_tot, H, D_v] FP32, gradient of the loss w.r.t. out
 *   d_final_state : [N, H, D_k, D_v] FP32 or NULL (zero), w.r.t. the final state
 *   dq, dk, dg    : [T_tot, H, D_k] FP32 outputs     dv : [T_tot, H, D_v] FP32
 *   dbeta         : [T_tot, H] FP32                 d_init_state : [N, H, D_k, D_v] or NULL
 *   workspace     : at least kda_backward_workspace_bytes(shape) bytes (for
 *                   the SIMT kernel: the state at every 4th token of every
 *                   unit and, for D_v > 32, the dq, dk, dg, dbeta parts of
 *                   value-column slices 2..)
 * q, k, v are BF16 or FP32 (shape->qkv_dtype); D_k, D_v in {32, 64, 128};
 * shape->chunk is ignored.  Every pointer 16-byte aligned; outputs must not
 * overlap inputs or each other.
 */
size_t kda_backward_workspace_bytes(const kda_shape *shape);
/* The backward kernel the last kda_backward call on this host thread
 * launched: 1 = chunked tensor-core, 0 = SIMT, -1 before the first launch. */
int kda_last_backward_path(void);
kda_status kda_backward(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *init_state, const int32_t *cu_seqlens,
                        const float *d_out, const float *d_final_state, float *dq, float *dk,
                        float *dv, float *dg, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, const kda_shape *shape, kda_stream_t stream);

/*
 * Affine state maps for context (sequence) parallelism.  The pages name KDA
 * context parallelism ("MoonshotAI/Kimi-K3 딥다이브", section 4-1) without
 * detail.  The recurrence is affine in its starting state: over a segment,
 * S_out = A S_in + B, with A the state of the segment run with v = 0 from the
 * identity and B its state from zero; token by token the outputs from S_in
 * are o_t(B) + S_in^T (A_t^T q_t), where A_t^T q_t is the output of the
 * v = 0, identity-start run.  (linear_attention_08_b200/cp.py combines the
 * segments of several ranks with these two calls.)
 *
 * kda_affine_rows:  y[r, h, :] = x[r, h, :] M[h]  (+ y when accumulate != 0)
 *   x : [rows, H, D_k]  y : [rows, H, D_v]  (shape->qkv_dtype, BF16 or FP32)
 *   M : [H, D_k, D_v] FP32.  y must not overlap x or M.
 * kda_affine_state: S_out[h] = A[h] S_in[h] + B[h]
 *   A : [H, D_k, D_k]  S_in, B, S_out : [H, D_k, D_v], all FP32; B may be NULL
 *   (zero); S_out may be exactly S_in or exactly B, but must not overlap A
 *   and must not partly overlap S_in or B (KDA_ERR_INVALID_ARGUMENT).
 * Only num_heads, head_dim_k, head_dim_v and qkv_dtype of the shape are used.
 */
kda_status kda_affine_rows(const void *x, const float *M, void *y, int64_t rows, int32_t accumulate,
                           const kda_shape *shape, kda_stream_t stream);
kda_status kda_affine_state(const float *A, const float *S_in, const float *B, float *S_out,
                            const kda_shape *shape, kda_stream_t stream);

/* Host helper: sum_i floor(T_i / ckpt_interval) for host int32 cu_seqlens[N+1]
 * (0 when ckpt_interval <= 0; -1 on a bad argument). */
int64_t kda_ckpt_count(const int32_t *host_cu_seqlens, int32_t num_seqs, int64_t ckpt_interval);

/* Workspace that lets kda_prefill_ws run this shape in a single window:
 * 74240 bytes per (chunk, head) packet for an upper bound of the chunk count
 * (every sequence may end in a partial chunk), plus one FP32 state per
 * (sequence, head) for the case without final_state.  0 for shapes off the
 * two-pass path, (size_t)-1 for an invalid shape. */
size_t kda_prefill_workspace_bytes(const kda_shape *shape);

/* Smallest workspace the two-pass path accepts (windows of one chunk);
 * 0 off that path, (size_t)-1 for an invalid shape. */
size_t kda_prefill_workspace_min_bytes(const kda_shape *shape);

/* Frees the memory cached by the library's per-device workspace pools. */
kda_status kda_release_workspace_pool(void);

/* Largest workspace kda_prefill takes from its pool, in bytes (default
 * 8 GiB), for calls made after this one on any thread.  Below
 * kda_prefill_workspace_min_bytes of a shape (with final_state: minus the
 * carried state), kda_prefill runs that shape on the single-pass kernel and
 * takes nothing from the pool; 0 therefore keeps the pool unused. */
kda_status kda_set_workspace_pool_cap(size_t bytes);

/* Which prefill kernel kda_prefill runs a shape on without explicit
 * positions, with an interval that is 0 or a multiple of 64 and the workspace
 * its pool cap allows:
 * 2 = two-pass tcgen05 tensor-core kernels (intra-chunk pass + chain): at most
 *     1024 sequences and 2048 (sequence, head) units, and only when the
 *     windows of chunks the workspace allows are worth it (below),
 * 1 = single-pass tcgen05 kernel (also used with explicit positions, without
 *     a workspace, for other intervals, and for larger batches, where its
 *     one CTA per (sequence, head) has the parallelism: from 4096 units on
 *     B200 it is the faster of the two),
 * 0 = SIMT FP32 kernel, -1 = invalid shape.
 * Windows: the host does not know the longest sequence, so a batch that does
 * not fit its workspace runs windows up to ceil(T_tot / 64) chunks, and those
 * past the longest sequence still cost both launches (about 5 us plus 6 ns
 * per unit each).  When that cost is over 5 % of the work (at about 35 M
 * tokens/s) and over 1 ms, kda_prefill and kda_prefill_ws run the single
 * pass instead. */
int kda_prefill_path(const kda_shape *shape);

/* The kernel (2, 1 or 0 as above) that the last kda_prefill,
 * kda_prefill_ws, kda_prefill_at or kda_prefill_noalloc call on this host
 * thread launched; -1 before the first launch.  Calls that return an error
 * before launching leave it unchanged. */
int kda_last_prefill_path(void);

/* Bounded-wait self-test: launches one CTA that waits on an mbarrier that
 * nothing arrives at, with the same bounded wait the tensor-core kernel
 * uses, giving up after max_polls polls.  The kernel writes
 * KDA_ERR_TIMEOUT to *dev_status and exits, so the context stays usable. */
kda_status kda_selftest_bounded_wait(int32_t *dev_status, int64_t max_polls,
                                     kda_stream_t stream);

/* The cudaError_t of the last KDA_ERR_CUDA on this thread. */
int kda_last_cuda_error(void);

const char *kda_status_string(kda_status status);

/* Library version as an integer: major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
