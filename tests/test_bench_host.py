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


def _tree(root, files):
    for rel, text in files.items():
        p = root / rel
        p.parent.mkdir(parents=True, exist_ok=True)
        p.write_text(text)


def test_source_digest_follows_includes(tmp_path, monkeypatch):
    """The digest that keys roofline.traffic covers a kernel source and every project header
    it reaches through includes, and nothing else."""
    csrc = "softmax_attn_sink_b200/csrc/"
    _tree(tmp_path, {csrc + "k.cu": '#include "a.cuh"\n#include <cuda.h>\nkernel\n',
                     csrc + "a.cuh": '#include "b.h"\na\n', "include/b.h": "b\n",
                     csrc + "other.cuh": "unrelated\n"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.source_digest("k.cu")
    (tmp_path / csrc / "other.cuh").write_text("changed\n")
    assert bench.source_digest("k.cu") == d0          # not included: no effect
    (tmp_path / "include/b.h").write_text("b changed\n")
    d1 = bench.source_digest("k.cu")
    assert d1 != d0                                   # reached through a.cuh
    (tmp_path / csrc / "k.cu").write_text('#include "a.cuh"\nkernel changed\n')
    assert bench.source_digest("k.cu") not in (d0, d1)


def test_kernel_traffic_only_for_the_measured_sources(tmp_path, monkeypatch):
    """profiles/traffic.txt's bytes are reported while the kernel's sources are the ones
    measured, and null once they change."""
    csrc = "softmax_attn_sink_b200/csrc/"
    _tree(tmp_path, {csrc + "k.cu": "kernel\n"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d = bench.source_digest("k.cu")
    _tree(tmp_path, {"profiles/traffic.txt": f"# comment k.cu 0 1\nk.cu  {d}  123456  capture\n"})
    assert bench.kernel_traffic("k.cu") == 123456
    assert bench.kernel_traffic("missing.cu") is None
    (tmp_path / csrc / "k.cu").write_text("kernel edited\n")
    assert bench.kernel_traffic("k.cu") is None
