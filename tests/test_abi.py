"""The C ABI: the library loads, exports every function include/attn_sink.h declares, and
rejects bad arguments on the host before touching the GPU.  CPU only (no compute calls)."""
import ctypes
import os
import re

import pytest

import softmax_attn_sink_b200 as sab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_sink.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_sink_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = sab.lib()
    declared = _declared_functions()
    assert "attn_sink_fwd" in declared and "attn_sink_bwd" in declared and "attn_sink_decode" in declared
    for name in declared:
        assert hasattr(L, name), f"{name} declared in attn_sink.h but not exported"
    assert set(sab._SYMBOLS) <= set(declared)


def test_debug_library_exports_the_same_symbols():
    """The bounds-checking build (libattn_sink_debug.so, built beside the release library)
    exports every declared function too, and ATTN_SINK_LIBRARY makes the binding load it."""
    import subprocess
    import sys
    from softmax_attn_sink_b200 import build as B
    if not os.path.exists(B.LIB_DEBUG):
        pytest.skip("debug library not built (python -m softmax_attn_sink_b200.build --debug)")
    D = ctypes.CDLL(B.LIB_DEBUG)
    for name in _declared_functions():
        assert hasattr(D, name), f"{name} missing from the debug library"
    code = "import softmax_attn_sink_b200 as s; s.lib(); print(s.LIB_PATH)"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       env=dict(os.environ, ATTN_SINK_LIBRARY=B.LIB_DEBUG), timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert os.path.samefile(r.stdout.strip().splitlines()[-1], B.LIB_DEBUG)


def test_params_struct_matches_header_field_order():
    text = open(HEADER).read()
    body = re.search(r"typedef struct \{(.*?)\} attn_sink_params;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\b([a-z_]+)\s*[;,]", body)
    assert names == [f[0] for f in sab.AttnSinkParams._fields_]


def test_status_strings_and_version():
    L = sab.lib()
    assert L.attn_sink_status_string(0) == b"ok"
    assert b"workspace" in L.attn_sink_status_string(3)
    assert L.attn_sink_status_string(99) == b"unknown status"
    assert L.attn_sink_version() == 0x000100


def _params(**kw):
    base = dict(batch=2, total_q=64, total_k=64, max_seqlen_q=32, max_seqlen_k=32, num_heads_q=8,
                num_heads_kv=2, head_dim_qk=128, head_dim_v=128, softmax_scale=0.088,
                causal=True, window_left=-1, window_right=-1, dtype=sab.ATTN_SINK_BF16)
    base.update(kw)
    return sab.make_params(**base)


SIZE_MAX = ctypes.c_size_t(-1).value


@pytest.mark.parametrize("bad,status", [
    (dict(num_heads_kv=3), 1), (dict(batch=0), 1), (dict(total_q=0), 1),
    (dict(head_dim_qk=96), 2), (dict(head_dim_v=256), 2), (dict(head_dim_qk=256), 2), (dict(dtype=7), 2),
    (dict(window_left=-2), 1), (dict(softmax_scale=float("inf")), 1),
    (dict(max_seqlen_q=0), 1), (dict(max_seqlen_k=65), 1),
])
def test_invalid_params_rejected_on_host(bad, status):
    L = sab.lib()
    p = _params(**bad)
    fake = 1 << 20  # never dereferenced: validation fails first
    st = L.attn_sink_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, None, None, 0, None)
    assert st == status
    assert L.attn_sink_fwd_workspace_size(ctypes.byref(p)) == SIZE_MAX


def test_null_and_misaligned_pointers_rejected():
    L = sab.lib()
    p = _params()
    a = 1 << 20
    assert L.attn_sink_fwd(ctypes.byref(p), None, a, a, a, a, None, a, None, None, 0, None) == 1
    assert L.attn_sink_fwd(ctypes.byref(p), a + 2, a, a, a, a, None, a, None, None, 0, None) == 1
    assert L.attn_sink_bwd(ctypes.byref(p), a, a, a, a, a, None, a, a, None, a, a, a, None,
                           None, 0, None) == 1  # lse is required


def test_bwd_workspace_is_required_and_sized():
    L = sab.lib()
    p = _params()
    need = L.attn_sink_bwd_workspace_size(ctypes.byref(p))
    # D + lse_tot (fp32 [Hq, T_q] each) + fp32 dQ accumulator [T_q, Hq, dk]
    assert need >= 2 * 8 * 64 * 4 + 64 * 8 * 128 * 4
    a = 1 << 20
    st = L.attn_sink_bwd(ctypes.byref(p), a, a, a, a, a, a, a, a, None, a, a, a, None, a, need - 256, None)
    assert st == 3
    st = L.attn_sink_bwd(ctypes.byref(p), a, a, a, a, a, a, a, a, None, a, a, a, None, None, 0, None)
    assert st == 3


def test_decode_params_and_workspace():
    L = sab.lib()
    p = _params(total_q=2, max_seqlen_q=1, total_k=40000, max_seqlen_k=30000)
    n = L.attn_sink_decode_num_splits(ctypes.byref(p))
    assert 1 <= n <= 1024
    ws = L.attn_sink_decode_workspace_size(ctypes.byref(p), 0)
    assert ws == L.attn_sink_decode_workspace_size(ctypes.byref(p), n)
    assert ws >= 2 * 8 * n * (128 + 2) * 4
    # decode needs total_q == batch and max_seqlen_q == 1
    bad = _params(total_q=3, max_seqlen_q=1)
    assert L.attn_sink_decode_workspace_size(ctypes.byref(bad), 0) == SIZE_MAX
    a = 1 << 20
    assert L.attn_sink_decode(ctypes.byref(p), a, a, a, a, None, -1, a, None, None, 0, None) == 1
    assert L.attn_sink_decode(ctypes.byref(p), a, a, a, a, None, 4, a, None, None, 0, None) == 3


def test_python_binding_requires_cuda_tensors():
    import torch
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        sab.attn_sink_fwd(q, q, q, cu, cu, 4, 4)


@pytest.mark.parametrize("change,status", [
    (dict(block_size=40), 1), (dict(block_size=8), 1), (dict(block_size=2048), 1),
    (dict(num_blocks=3), 1), (dict(max_blocks=0), 1), (dict(table=None), 1),
    (dict(dtype=sab.ATTN_SINK_FP32), 2), (dict(total_q=5), 1),
])
def test_paged_decode_rejects_bad_arguments_on_host(change, status):
    """The paged decode validates its table shape and block size before any launch (fake,
    aligned, non-null device addresses: nothing is dereferenced)."""
    a = dict(block_size=16, num_blocks=4, max_blocks=2, table=256, dtype=sab.ATTN_SINK_BF16, total_q=2)
    a.update(change)
    p = _params(batch=2, total_q=a["total_q"], total_k=64, max_seqlen_q=1, max_seqlen_k=32,
                dtype=a["dtype"])
    fake = 4096
    st = sab.lib().attn_sink_decode_paged(ctypes.byref(p), fake, fake, fake, a["table"], fake,
                                          a["num_blocks"], a["block_size"], a["max_blocks"], None, 0,
                                          fake, None, fake, 1 << 20, None)
    assert st == status


def test_check_seqlens_rejects_null_arrays_on_host():
    p = _params()
    assert sab.lib().attn_sink_check_seqlens(ctypes.byref(p), None, None, None) == 1
    assert sab.lib().attn_sink_check_seqlens(None, None, 4096, None) == 1


@pytest.mark.parametrize("drop,change,status", [
    (None, {}, 1),                                    # NULL dropout
    ((1.0, 1, 0), {}, 1), ((-0.1, 1, 0), {}, 1),      # p out of range (T = 0, T > 256)
    ((float("nan"), 1, 0), {}, 1),
    ((0.1, 1, 0), dict(dtype=sab.ATTN_SINK_FP32), 2),  # tensor-core path only
])
def test_dropout_entry_points_validate_on_host(drop, change, status):
    """attn_sink_fwd_dropout / attn_sink_bwd_dropout reject a missing or out-of-range dropout
    and unsupported dtypes before any launch (fake, aligned device addresses)."""
    L = sab.lib()
    p = _params(**change)
    d = None if drop is None else ctypes.byref(sab.AttnSinkDropout(*drop))
    a = 1 << 20
    ws = L.attn_sink_bwd_workspace_size(ctypes.byref(p))
    assert L.attn_sink_fwd_dropout(ctypes.byref(p), a, a, a, a, a, None, d, a, None, None, 0,
                                   None) == status
    assert L.attn_sink_bwd_dropout(ctypes.byref(p), a, a, a, a, a, a, a, a, None, d, a, a, a, None,
                                   a, ws, None) == status


def test_dropout_struct_matches_header():
    text = open(HEADER).read()
    body = re.search(r"typedef struct \{([^{}]*)\} attn_sink_dropout;", text).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\b([a-z_]+)\s*;", body)
    assert names == [f[0] for f in sab.AttnSinkDropout._fields_]
    assert ctypes.sizeof(sab.AttnSinkDropout) == 24


def test_fwd_workspace_size():
    """The forward's workspace holds the work counter of the persistent tensor-core kernel."""
    L = sab.lib()
    assert L.attn_sink_fwd_workspace_size(ctypes.byref(_params())) == 256


@pytest.mark.gpu
def test_tensor_core_fwd_requires_its_workspace():
    """Without the workspace attn_sink_fwd_workspace_size() asks for, the tensor-core
    forward returns ATTN_SINK_ERR_WORKSPACE before any launch; with it, it runs."""
    import torch
    L = sab.lib()
    q = torch.randn(64, 8, 128, device="cuda").to(torch.bfloat16)
    k = torch.randn(64, 2, 128, device="cuda").to(torch.bfloat16)
    cu = torch.tensor([0, 32, 64], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    p = _params()
    stream = torch.cuda.current_stream().cuda_stream
    args = (ctypes.byref(p), q.data_ptr(), k.data_ptr(), k.data_ptr(), cu.data_ptr(), cu.data_ptr(), None,
            out.data_ptr(), None)
    assert L.attn_sink_fwd(*args, None, 0, stream) == 3
    ws = torch.empty(L.attn_sink_fwd_workspace_size(ctypes.byref(p)), dtype=torch.uint8, device="cuda")
    assert L.attn_sink_fwd(*args, ws.data_ptr(), ws.numel() - 16, stream) == 3
    assert L.attn_sink_fwd(*args, ws.data_ptr(), ws.numel(), stream) == 0
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
