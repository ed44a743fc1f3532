"""attn_sink_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a custom-op host that offers no allocator, a process whose memory is all
held by another pool, a loop that must not allocate).  It keeps its chunk partials in a
fixed 16 MiB array inside the library instead of a caller workspace.

Called through the C ABI with ctypes.  Its results must match attn_sink_decode's on the
same inputs, within the bf16 tolerances the other tests use, on two calls in a row (the
second call reuses the array the first one left behind).  The file name sorts last so
that a run stopping at the first failure has already run every other test."""
import ctypes

import pytest

import workloads as W
from _check import check_lse, check_out, to_np

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
    p = _params(d, q, k, v, max_k)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = f(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.data_ptr(),
               sink.data_ptr(), num_splits, out.data_ptr(), lse.data_ptr(), stream)
        assert st == 0, sab.lib().attn_sink_status_string(st)
        torch.cuda.synchronize()
        check_out(to_np(out), to_np(ref_out), "bf16", f"out (call {call + 1})")
        check_lse(to_np(lse), to_np(ref_lse), "bf16", f"lse (call {call + 1})")


def test_noalloc_decode_rejects_partials_beyond_the_fixed_array():
    import torch
    import softmax_attn_sink_b200 as sab
    f = _noalloc_fn()
    d = W.random_decode(42, [64, 64], hq=16, hkv=2, dk=128, dv=128)
    q, k, v, cu, sink = _inputs(d)
    p = _params(d, q, k, v, 64)
    per_split = 2 * 16 * (128 + 2) * 4
    too_many = SCRATCH_BYTES // per_split + 8
    out = torch.empty(2, 16, 128, dtype=torch.bfloat16, device="cuda")
    st = f(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.data_ptr(),
           sink.data_ptr(), too_many, out.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert st == 3  # ATTN_SINK_ERR_WORKSPACE, returned before any launch
