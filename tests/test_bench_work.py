"""bench.py's algorithmic work accounting against hand counts on a tiny labelled problem:
sparse FLOPs count only the valid rows and keys of critical pairs (ragged tails included),
the aggregation credits min(#marginal, #non-marginal) states per query block, and the
algorithmic bytes are Q, K, V read and O written once plus the labels and alpha."""

import types

import torch

import bench


def test_work_of_a_ragged_labelled_problem():
    # N = 150, block_q = 64 (query blocks of 64, 64, 22 rows), block_kv = 64 (64, 64, 22 keys)
    w = types.SimpleNamespace(B=1, H=1, N=150, D=8, block_q=64, block_kv=64)
    mask = torch.tensor([[[[2, 1, 0],
                           [1, 1, 2],
                           [2, 2, 1]]]], dtype=torch.int8)
    work = bench.algorithmic_work(w, mask)
    D, N = 8, 150
    # critical pairs (rows x keys): (64 x 64) + (64 x 22) + (22 x 64) + (22 x 64)
    pairs = 64 * 64 + 64 * 22 + 22 * 64 + 22 * 64
    assert work["f_sparse"] == 4 * D * pairs
    # marginal counts per row: 1, 2, 1 -> min(m, 3 - m) = 1, 1, 1
    assert work["f_agg"] == 3 * D * D
    assert work["f_states"] == 2 * N * D * D
    assert work["f_attn_kernel"] == 4 * D * pairs + 2 * N * D * D
    assert work["f_router"] == 2 * (N * D + 3 * 3 * D)
    # backward: five products per critical pair, four D x D products per row, the aggregation
    assert work["f_bwd"] == 10 * D * pairs + 4 * N * D * D + 3 * D * D + 8 * N * D
    # PISA: non-critical blocks per row 2, 2, 1 over rows of 64, 64, 22
    assert work["f_pisa"] == 4 * D * pairs + 4 * D * (64 * 2 + 64 * 2 + 22 * 1) + 4 * N * D * D
    expected = 4 * D * pairs + 2 * N * D * D + 2 * N * D * D + 3 * D * D + 2 * (N * D + 9 * D) + 3 * N * D
    assert work["flops"] == expected
    assert work["bytes"] == 8 * N * D + 9 + 1 * D * 4


def test_dense_equivalent_flops():
    w = types.SimpleNamespace(B=2, H=3, N=100, D=64)
    assert bench.dense_equivalent_flops(w) == 4.0 * 2 * 3 * 100 ** 2 * 64
