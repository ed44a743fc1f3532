"""attn_sink_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a custom-op host that offers no allocator, a process whose memory is all
held by another pool, a loop that must not allocate).  It keeps its chunk partials in a
fixed 16 MiB array inside the library instead of a caller workspace.

Called through the C ABI with ctypes.  Its results must match attn_sink_decode's on the
same inputs, within the bf16 tolerances the other tests use, on two calls in a row (the
second call reuses the array the first one left behind), and the oracle's decode.  The
file name sorts last so that a run stopping at the first failure has already run every
other test."""
import ctypes

import numpy as np
import pytest

import workloads as W
from _check import check_lse, check_out, to_np
from oracle import ref

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _noalloc_fn():
    import softmax_attn_sink_b200 as sab
    f = sab.lib().attn_sink_decode_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(sab.AttnSinkParams), vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _inputs(d):
    import torch
    td = torch.bfloat16
    return (torch.from_numpy(d.q).cuda().to(td), torch.from_numpy(d.k).cuda().to(td),
            torch.from_numpy(d.v).cuda().to(td), torch.from_numpy(d.cu_seqlens_k).cuda(),
            torch.from_numpy(d.sink).cuda())


def _params(d, q, k, v, max_k):
    import softmax_attn_sink_b200 as sab
    return sab.make_params(batch=q.shape[0], total_q=q.shape[0], total_k=k.shape[0],
                           max_seqlen_q=1, max_seqlen_k=max_k, num_heads_q=q.shape[1],
                           num_heads_kv=k.shape[1], head_dim_qk=q.shape[2],
                           head_dim_v=v.shape[2], softmax_scale=d.softmax_scale, causal=True)


def _call(f, p, q, k, v, cu, sink, num_splits, out, lse):
    import torch
    return f(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.data_ptr(),
             sink.data_ptr(), num_splits, out.data_ptr(), None if lse is None else lse.data_ptr(),
             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("num_splits,dim", [(0, 128), (5, 128), (0, 256)])
def test_noalloc_decode_matches_workspace_decode_twice(num_splits, dim):
    import torch
    import softmax_attn_sink_b200 as sab
    f = _noalloc_fn()
    d = W.random_decode(41, [3000, 1, 777, 5000], hq=16, hkv=2, dk=dim, dv=dim)
    q, k, v, cu, sink = _inputs(d)
    max_k = 5000
    ref_out, ref_lse = sab.attn_sink_decode(q, k, v, cu, max_k, sink, d.softmax_scale, True,
                                            (-1, -1), num_splits)
    ro, rl = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale)
    p = _params(d, q, k, v, max_k)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _call(f, p, q, k, v, cu, sink, num_splits, out, lse)
        assert st == 0, sab.lib().attn_sink_status_string(st)
        torch.cuda.synchronize()
        check_out(to_np(out), to_np(ref_out), "bf16", f"out (call {call + 1})")
        check_lse(to_np(lse), to_np(ref_lse), "bf16", f"lse (call {call + 1})")
        # and against the oracle directly
        check_out(to_np(out), ro, "bf16", f"out vs oracle (call {call + 1})")
        check_lse(to_np(lse), rl, "bf16", f"lse vs oracle (call {call + 1})")


# 64 sequences x 64 q heads: with one 2048-key sequence the automatic count is 8 splits of
# 256 keys, whose partials (4096 rows x 8 splits x 520 bytes) need just over 16 MiB.
_BIG_LENS = [2048] + [int(n) for n in np.random.default_rng(44).integers(1, 400, size=63)]


def _largest_fitting(lib, p, upto):
    best = 0
    for s in range(1, upto + 1):
        if lib.attn_sink_decode_workspace_size(ctypes.byref(p), s) <= SCRATCH_BYTES:
            best = s
    return best


def test_noalloc_decode_lowers_the_automatic_split_count_to_fit():
    import torch
    import softmax_attn_sink_b200 as sab
    L = sab.lib()
    f = _noalloc_fn()
    d = W.random_decode(43, _BIG_LENS, hq=64, hkv=8, dk=128, dv=128)
    q, k, v, cu, sink = _inputs(d)
    p = _params(d, q, k, v, 2048)
    auto = L.attn_sink_decode_num_splits(ctypes.byref(p))
    assert L.attn_sink_decode_workspace_size(ctypes.byref(p), auto) > SCRATCH_BYTES
    fit = _largest_fitting(L, p, auto)
    assert 1 <= fit < auto
    ref_out, ref_lse = sab.attn_sink_decode(q, k, v, cu, 2048, sink, d.softmax_scale, True,
                                            (-1, -1), fit)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _call(f, p, q, k, v, cu, sink, 0, out, lse)
        assert st == 0, L.attn_sink_status_string(st)
        torch.cuda.synchronize()
        # the same kernels with the same split count: the same bits
        assert torch.equal(out, ref_out), f"out differs from attn_sink_decode (call {call + 1})"
        assert torch.equal(lse, ref_lse), f"lse differs from attn_sink_decode (call {call + 1})"
    o, l = to_np(out), to_np(lse)
    for b in (0, 1, 63):
        k0, k1 = int(d.cu_seqlens_k[b]), int(d.cu_seqlens_k[b + 1])
        for g in (0, 5):
            heads = list(range(g * 8, g * 8 + 8))
            ro, rl = ref.decode(d.q[b:b + 1, heads], d.k[k0:k1, g:g + 1], d.v[k0:k1, g:g + 1],
                                np.array([0, k1 - k0]), d.sink[heads], d.softmax_scale)
            check_out(o[b, heads], ro[0], "bf16", f"out[b={b},g={g}] vs oracle")
            check_lse(l[heads, b], rl[:, 0], "bf16", f"lse[b={b},g={g}] vs oracle")


def test_noalloc_decode_rejects_partials_beyond_the_fixed_array():
    import torch
    import softmax_attn_sink_b200 as sab
    L = sab.lib()
    f = _noalloc_fn()
    d = W.random_decode(43, _BIG_LENS, hq=64, hkv=8, dk=128, dv=128)
    q, k, v, cu, sink = _inputs(d)
    p = _params(d, q, k, v, 2048)
    # the smallest explicit count whose partials (by the library's own sizing) exceed 16 MiB
    first_over = next(s for s in range(1, 4096)
                      if L.attn_sink_decode_workspace_size(ctypes.byref(p), s) > SCRATCH_BYTES)
    out = torch.full((64, 64, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((64, 64), float("nan"), dtype=torch.float32, device="cuda")
    st = _call(f, p, q, k, v, cu, sink, first_over, out, lse)
    assert st == 3  # ATTN_SINK_ERR_WORKSPACE, returned before any launch
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all(), "a rejected call wrote its outputs"
    st = _call(f, p, q, k, v, cu, sink, first_over - 1, out, lse)
    assert st == 0, L.attn_sink_status_string(st)
    torch.cuda.synchronize()
    ref_out, ref_lse = sab.attn_sink_decode(q, k, v, cu, 2048, sink, d.softmax_scale, True,
                                            (-1, -1), first_over - 1)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
