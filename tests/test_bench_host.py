"""Host-side helpers of bench.py (no GPU): the diagonal-block count behind
the prefill's causal-effective FLOPs, and the host CPU record."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_diagonal_blocks_counts_rows_holding_their_own_tile():
    T = 4  # units u = h * T + t
    idx = torch.full((2 * T, 3), -1, dtype=torch.int32)
    idx[0, 0] = 0                           # t = 0: diagonal
    idx[1, 0] = 0                           # t = 1: sink only
    idx[2, :2] = torch.tensor([0, 2])       # t = 2: diagonal
    idx[3, 0] = 2                           # t = 3: no
    idx[4, 0] = 0                           # t = 0: diagonal
    idx[5, :2] = torch.tensor([0, 1])       # t = 1: diagonal
    idx[6, 0] = 5                           # t = 2: no
    idx[7, 2] = 3                           # t = 3: diagonal, last slot
    assert bench.diagonal_blocks(idx, T) == 5


def test_diagonal_blocks_of_dense_causal_lists():
    T = 6
    rows = []
    for t in range(T):
        rows.append(list(range(t + 1)) + [-1] * (T - t - 1))
    idx = torch.tensor(rows, dtype=torch.int32)
    assert bench.diagonal_blocks(idx, T) == T


def test_host_cpu_model_is_a_string():
    m = bench.host_cpu_model()
    assert isinstance(m, str)
    if os.path.exists("/proc/cpuinfo"):
        assert m
