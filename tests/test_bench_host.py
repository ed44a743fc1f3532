"""Host logic of bench.py: its algorithmic-work counter agrees with the oracle's mask."""
import numpy as np
import pytest

import bench
import workloads as W
from oracle import ref


@pytest.mark.parametrize("causal,wl,wr", [(True, -1, -1), (False, -1, -1), (True, 5, -1),
                                          (False, 3, 2), (False, -1, 0)])
def test_visible_pairs_matches_oracle(causal, wl, wr):
    cu_q = np.array([0, 3, 8, 8, 20], dtype=np.int32)
    cu_k = np.array([0, 5, 7, 9, 21], dtype=np.int32)
    assert bench.visible_pairs(cu_q, cu_k, 3, causal, wl, wr) == ref.pair_count(cu_q, cu_k, 3, causal, wl, wr)


def test_headline_workload_pairs():
    L = W.config2_lengths().astype(np.int64)
    cu = W.cu_from_lengths(L)
    n = bench.visible_pairs(cu, cu, 32, True)
    assert n == 32 * int((L * (L + 1) // 2).sum())
    p4 = W.config4(1.0)
    assert bench.visible_pairs(p4.cu_seqlens_q, p4.cu_seqlens_k, 1, True, 512, 0) == \
        ref.pair_count(p4.cu_seqlens_q, p4.cu_seqlens_k, 1, True, 512, 0)
