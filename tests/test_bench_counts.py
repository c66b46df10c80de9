"""The work counts bench.py divides by, checked by brute force on small
shapes: the chunkwise form's FLOPs (every score of a chunk's block, and only
its causal half) and the algorithmic bytes of the forward."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _chunk_flops(C, dk, dv, causal):
    """FLOPs of one full chunk of C tokens, counted operation by operation:
    scores q_r . k_c (2 dk each), P V (2 dv per score), the read-out q_r^T R
    (2 dk dv per row) and the state update K^T V (2 dk dv per row)."""
    total = 0
    for r in range(C):
        cols = r + 1 if causal else C
        total += cols * 2 * dk      # scores of row r
        total += cols * 2 * dv      # row r of P V
        total += 2 * dk * dv        # read-out of row r
        total += 2 * dk * dv        # row r's share of K^T V
    return total


def test_flop_counts_match_brute_force():
    for C, dk, dv in ((4, 2, 3), (16, 16, 16), (64, 64, 64), (128, 256, 512)):
        assert bench.flops_per_token_head(C, dk, dv) * C == _chunk_flops(C, dk, dv, causal=False)
        assert bench.flops_per_token_head_causal(C, dk, dv) * C == _chunk_flops(C, dk, dv, causal=True)


def test_algorithmic_bytes_of_the_headline_workload():
    w = dict(bench.WORKLOAD)
    B, N, H, dk, dv = w["B"], w["N"], w["H"], w["dk"], w["dv"]
    tok = B * N * H
    # q, k, v read once (bf16), out written once (bf16), the fp32 final state
    expect = tok * dk * 2 * 2 + tok * dv * 2 + tok * dv * 2 + B * H * dk * dv * 4
    assert bench.algo_bytes(w, out_bytes=2) == expect == 411041792
