"""Host-side pieces of bench.py, on the CPU: the algorithmic byte counts behind
every roofline figure, and the expert folding of the GEMM legs' small cases."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402


def test_decode_algorithmic_bytes_by_hand():
    """Decode (R=8, T=128, H=7168, K=8, E=256, e4m3 per 128, every entry valid):
    dispatch reads x (2H) and the routing (8K + 4K) per token and writes each
    entry's codes, fp32 scales (4 * H/128) and source info (4); combine reads
    every entry's bf16 row (2H), the routing, weights and slots, and writes the
    bf16 output."""
    w = synth.workload("decode")
    idx, _ = synth.make_routing(w)
    N, K, H = 1024, 8, 7168
    assert (idx >= 0).all() and idx.shape == (N, K)
    b, v = bench.algorithmic_bytes(w, "e4m3_b128", idx)
    assert v == N * K
    assert b["dispatch"] == N * (2 * H + 8 * K + 4 * K) + v * (H + 4 * (H // 128) + 4)
    assert b["combine"] == v * 2 * H + N * (8 * K + 4 * K + 4 * K + 2 * H)
    assert b["layout"] == N * (8 * K + 4 * K + 8)


def test_masked_entries_move_no_rows():
    w = synth.workload("tiny")
    idx, _ = synth.make_routing(w)
    all_masked = np.full_like(idx, -1)
    b, v = bench.algorithmic_bytes(w, "bf16", all_masked)
    assert v == 0
    N, K, H = w["N"], w["K"], w["H"]
    assert b["dispatch"] == N * (2 * H + 8 * K + 4 * K)
    assert b["combine"] == N * (8 * K + 4 * K + 4 * K + 2 * H)


def test_gemm_routing_folds_experts_and_keeps_masked_entries():
    class A:
        gemm_experts = 32
    idx = torch.tensor([[0, 33, 255, -1], [31, 32, 64, 7]], dtype=torch.int64)
    E, folded = bench.gemm_routing(256, idx, A())
    assert E == 32
    assert folded.tolist() == [[0, 1, 31, -1], [31, 0, 0, 7]]

    class B:
        gemm_experts = 0
    E, same = bench.gemm_routing(256, idx, B())
    assert E == 256 and same is idx
