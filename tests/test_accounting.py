"""The benchmark's algorithmic counts reproduce the pages' cost formulas."""
import os

import bench

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "cost_counts.txt")


def rows():
    with open(GOLDEN) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                name, C, D, value = line.split()
                yield name, int(C), int(D), int(value)


def test_cost_formulas_match_golden():
    seen = 0
    for name, C, D, value in rows():
        if name == "decode_flops_per_head_token":
            assert bench.decode_flops_per_token_head(D) == value
        elif name == "decode_state_bytes_per_head_token":
            assert bench.decode_state_bytes_per_token_head(D, D) == value
        elif name == "prefill_flops_per_chunk":
            assert bench.prefill_flops_per_chunk(C, D) == value
        seen += 1
    assert seen == 5


def test_prefill_workload_totals():
    # B=4, T=8192, H=32, D=128, C=64: 512 chunks x 32 heads
    flops, byts = bench.prefill_algorithmic([8192] * 4, 32, 128, 128, 64, 2, 0, False)
    assert flops == 512 * 32 * 13631488
    # 1,540 bytes per token-head (bf16 q, k, v, o; fp32 g and beta) + the final state
    assert bench.prefill_io_bytes_per_token_head(128, 128, 2) == 1540
    assert byts == 32768 * 32 * 1540 + 4 * 32 * 128 * 128 * 4
