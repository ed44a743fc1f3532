"""Guard regions around every output buffer: a store past either end of out, lse, dq, dk,
dv, dsink or a decode output would go unseen by tests that read only the tensors' own
elements.  Each output here is a view into a larger device buffer filled with 0xFF bytes,
whose leading and trailing 4 KB are guards; after the call both guards must be intact, and
no element of the output may still be all ones (every element must be written, including
the zeros of rows or keys that see nothing).  All-ones is a NaN in bf16, fp16 and fp32,
which no correct output is.  Values are compared with the oracle as well, and the device
status word must stay clear.  test_debug_build.py runs this file again against the
bounds-checking debug library.

The cu_seqlens contract is the caller's (CANN flash_attn doc, "SeqLengths Parameter
Group"); with valid cu_seqlens every kernel must stay inside its outputs.  The cases span
varlen GQA with empty sequences and sq != sk, the persistent forward with and without
its output staging area, the one-CTA-per-item grid forward, head dims 64 / 128 / 256 and
dv 32, fp16 and fp32, dropout, the atomic, deterministic and dropout backward, and the
packed and paged decode."""
import os

import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_grad, check_lse, check_out, to_np

pytestmark = pytest.mark.gpu

try:
    import torch
    import softmax_attn_sink_b200 as sab
    from gpu_util import dev, tdtype, window
except Exception:  # torch without CUDA still imports; the calls fail at run time
    pass

GUARD = 4096
PATTERN = 0xFF


class Guarded:
    """A contiguous tensor of `shape` inside a byte buffer with guard regions on both sides."""

    def __init__(self, shape, dtype, what):
        esize = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * esize
        self.esize, self.what = esize, what
        self.raw = torch.full((GUARD + self.n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.n].view(dtype).view(*shape)

    def check(self):
        torch.cuda.synchronize()
        head, tail = self.raw[:GUARD], self.raw[GUARD + self.n:]
        assert bool((head == PATTERN).all()), f"{self.what}: bytes before the buffer were written"
        assert bool((tail == PATTERN).all()), f"{self.what}: bytes after the buffer were written"
        body = self.raw[GUARD:GUARD + self.n].view(-1, self.esize)
        untouched = (body == PATTERN).all(dim=1)
        assert not bool(untouched.any()), \
            f"{self.what}: {int(untouched.sum())} elements were never written"


_LENS_D = [int(n) for n in np.random.default_rng(43).integers(0, 300, size=600)]
_LENS_C = [int(n) for n in np.random.default_rng(13).integers(0, 5, size=9000)]

FWD_CASES = [
    # name, lens_q, lens_k, hq, hkv, dk, dv, causal, wl, wr, dtype, dropout p
    ("staged_varlen_gqa", [1, 127, 0, 129, 333], [1, 127, 0, 129, 333], 8, 2, 128, 128, True, -1, -1,
     "bf16", None),
    ("sq_ne_sk_odd_group", [5, 100, 200, 7], [2, 300, 150, 0], 3, 1, 128, 64, True, -1, -1, "bf16", None),
    ("unstaged_600_sequences", _LENS_D, _LENS_D, 4, 2, 128, 128, True, -1, -1, "bf16", None),
    ("grid_9000_sequences", _LENS_C, _LENS_C, 2, 1, 128, 128, True, -1, -1, "bf16", None),
    ("dk64_window", [300, 129], [333, 200], 2, 1, 64, 64, True, 100, 0, "bf16", None),
    ("dk64_dv32_window", [300, 129, 0], [333, 200, 5], 2, 1, 64, 32, True, 100, 0, "bf16", None),
    ("d256_varlen", [1, 65, 0, 300], [1, 65, 0, 333], 4, 2, 256, 256, True, -1, -1, "bf16", None),
    ("fp16", [200, 3], [260, 300], 4, 4, 128, 64, True, -1, -1, "fp16", None),
    ("fp32", [70, 1, 130], [90, 5, 130], 4, 2, 128, 64, True, -1, -1, "fp32", None),
    ("dropout", [300, 129, 0, 257], [300, 129, 0, 257], 8, 2, 128, 128, True, -1, -1, "bf16", 0.2),
]


def _status_clear():
    """No kernel set a status bit (in the debug library: no store left its output)."""
    assert sab.device_status() == (0, 0)


@pytest.fixture(autouse=True)
def _fresh_status():
    sab.device_status()   # read and clear whatever an earlier test left
    yield


def test_library_in_use():
    """Run with ATTN_SINK_EXPECT_LIBRARY set (the debug-library run), the package must have
    loaded that file."""
    want = os.environ.get("ATTN_SINK_EXPECT_LIBRARY")
    sab.lib()
    if want:
        assert os.path.samefile(sab.LIB_PATH, want)


def _fwd_guarded(p, dropout):
    td = tdtype(p)
    q, k, v = dev(p.q, td), dev(p.k, td), dev(p.v, td)
    cu_q, cu_k = dev(p.cu_seqlens_q), dev(p.cu_seqlens_k)
    sink = None if p.sink is None else dev(p.sink)
    go = Guarded((q.shape[0], q.shape[1], v.shape[2]), td, "out")
    gl = Guarded((q.shape[1], q.shape[0]), torch.float32, "lse")
    sab.attn_sink_fwd(q, k, v, cu_q, cu_k, max(p.max_seqlen_q, 1), max(p.max_seqlen_k, 1), sink,
                      p.softmax_scale, p.causal, window(p), out=go.t, lse=gl.t, dropout=dropout)
    return (q, k, v, cu_q, cu_k, sink), go, gl


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fwd_stays_inside_its_outputs(case):
    name, lq, lk, hq, hkv, dk, dv, causal, wl, wr, dtype, pdrop = case
    p = W.random_problem(len(name) * 31 + hq, lq, lk, hq, hkv, dk, dv, causal, wl, wr, "normal", dtype)
    drop = None if pdrop is None else (pdrop, 0x1234567890ABCDEF, 5)
    _, go, gl = _fwd_guarded(p, drop)
    go.check()
    gl.check()
    _status_clear()
    ro, rl = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                     p.causal, wl, wr, dropout=drop)
    check_out(to_np(go.t), ro, dtype)
    check_lse(to_np(gl.t), rl, dtype)


BWD_CASES = [
    # name, lens_q, lens_k, hq, hkv, dk, dv, causal, wl, wr, dtype, mode
    ("atomic_varlen_gqa", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 128, 128, True, -1, -1, "bf16", "atomic"),
    ("atomic_sq_ne_sk_window", [5, 130, 260], [2, 200, 300], 4, 2, 128, 128, True, 50, 0, "bf16", "atomic"),
    ("deterministic_varlen", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 128, 128, True, -1, -1, "bf16",
     "deterministic"),
    ("dropout_varlen", [1, 129, 0, 257], [1, 129, 0, 257], 4, 2, 128, 128, True, -1, -1, "bf16", "dropout"),
    ("dk64_sq_ne_sk", [5, 130], [2, 200], 4, 2, 64, 64, True, -1, -1, "bf16", "atomic"),
    ("dk64_dv32_window", [300, 129, 0], [333, 200, 5], 2, 1, 64, 32, True, 100, 0, "bf16", "atomic"),
    ("d256_varlen", [1, 65, 0, 300], [1, 65, 0, 333], 4, 2, 256, 256, True, -1, -1, "bf16", "atomic"),
    ("fp16_atomic", [300, 200], [300, 200], 4, 4, 128, 128, True, -1, -1, "fp16", "atomic"),
    ("fp32", [70, 1, 130], [90, 5, 130], 4, 2, 128, 64, True, -1, -1, "fp32", "atomic"),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_stays_inside_its_outputs(case):
    name, lq, lk, hq, hkv, dk, dv, causal, wl, wr, dtype, mode = case
    p = W.random_problem(len(name) * 17 + hq, lq, lk, hq, hkv, dk, dv, causal, wl, wr, "normal", dtype,
                         with_dout=True)
    drop = (0.2, 0xFEDCBA9876543210, 9) if mode == "dropout" else None
    (q, k, v, cu_q, cu_k, sink), go, gl = _fwd_guarded(p, drop)
    go.check()
    gl.check()
    td = tdtype(p)
    gq = Guarded(tuple(q.shape), td, "dq")
    gk = Guarded(tuple(k.shape), td, "dk")
    gv = Guarded(tuple(v.shape), td, "dv")
    gs = Guarded((q.shape[1],), torch.float32, "dsink")
    sab.attn_sink_bwd(q, k, v, go.t, dev(p.dout, td), gl.t, cu_q, cu_k, max(p.max_seqlen_q, 1),
                      max(p.max_seqlen_k, 1), sink, p.softmax_scale, p.causal, window(p), dq=gq.t,
                      dk=gk.t, dv=gv.t, dsink=gs.t, deterministic=mode == "deterministic", dropout=drop)
    for g in (gq, gk, gv, gs):
        g.check()
    _status_clear()
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, p.causal, wl, wr)
    rdq, rdk, rdv, rds = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=drop)
    check_grad(to_np(gq.t), rdq, dtype, "dq")
    check_grad(to_np(gk.t), rdk, dtype, "dk")
    check_grad(to_np(gv.t), rdv, dtype, "dv")
    check_grad(to_np(gs.t), rds, dtype, "dsink")


@pytest.mark.parametrize("dim,splits", [(128, 0), (128, 7), (256, 0)])
def test_decode_stays_inside_its_outputs(dim, splits):
    d = W.random_decode(61 + dim, [3000, 1, 0, 777, 5000], hq=16, hkv=2, dk=dim, dv=dim)
    td = torch.bfloat16
    q, k, v = dev(d.q, td), dev(d.k, td), dev(d.v, td)
    cu, sink = dev(d.cu_seqlens_k), dev(d.sink)
    go = Guarded((5, 16, dim), td, "out")
    gl = Guarded((16, 5), torch.float32, "lse")
    sab.attn_sink_decode(q, k, v, cu, 5000, sink, d.softmax_scale, True, (-1, -1), splits,
                         out=go.t, lse=gl.t)
    go.check()
    gl.check()
    _status_clear()
    ro, rl = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale)
    check_out(to_np(go.t), ro, "bf16")
    check_lse(to_np(gl.t), rl, "bf16")


def test_paged_decode_stays_inside_its_outputs():
    lens = [3000, 1, 0, 777, 5000]
    d = W.random_decode(71, lens, hq=16, hkv=2, dk=128, dv=128)
    table, nb = W.paged_layout(72, lens, 64)
    kc = W.to_paged(d.k, d.cu_seqlens_k, table, 64, nb)
    vc = W.to_paged(d.v, d.cu_seqlens_k, table, 64, nb)
    used = np.array(lens, np.int32)
    td = torch.bfloat16
    go = Guarded((5, 16, 128), td, "out")
    gl = Guarded((16, 5), torch.float32, "lse")
    sab.attn_sink_decode_paged(dev(d.q, td), dev(kc, td), dev(vc, td), dev(table), dev(used), 5000,
                               dev(d.sink), d.softmax_scale, out=go.t, lse=gl.t)
    go.check()
    gl.check()
    _status_clear()
    ro, rl = ref.decode_paged(d.q, kc, vc, table, used, 64, d.sink, d.softmax_scale)
    check_out(to_np(go.t), ro, "bf16")
    check_lse(to_np(gl.t), rl, "bf16")
