"""Helpers for the GPU parity tests: move a seeded problem to the device, run the
library through its Python binding (which calls the C ABI), bring results back."""
import numpy as np
import torch

import softmax_attn_sink_b200 as sab


def tdtype(p):
    return {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[p.dtype]


def dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t if dtype is None else t.to(dtype)


def window(p):
    return (p.window_left, p.window_right)


def run_fwd(p, dropout=None):
    td = tdtype(p)
    q, k, v = dev(p.q, td), dev(p.k, td), dev(p.v, td)
    cu_q, cu_k = dev(p.cu_seqlens_q), dev(p.cu_seqlens_k)
    sink = None if p.sink is None else dev(p.sink)
    out, lse = sab.attn_sink_fwd(q, k, v, cu_q, cu_k, max(p.max_seqlen_q, 1), max(p.max_seqlen_k, 1),
                                 sink, p.softmax_scale, p.causal, window(p), dropout=dropout)
    torch.cuda.synchronize()
    return out, lse


def run_bwd(p, deterministic=False, dropout=None):
    td = tdtype(p)
    q, k, v = dev(p.q, td), dev(p.k, td), dev(p.v, td)
    do = dev(p.dout, td)
    cu_q, cu_k = dev(p.cu_seqlens_q), dev(p.cu_seqlens_k)
    sink = None if p.sink is None else dev(p.sink)
    mq, mk = max(p.max_seqlen_q, 1), max(p.max_seqlen_k, 1)
    out, lse = sab.attn_sink_fwd(q, k, v, cu_q, cu_k, mq, mk, sink, p.softmax_scale, p.causal, window(p),
                                 dropout=dropout)
    dq, dk, dv, ds = sab.attn_sink_bwd(q, k, v, out, do, lse, cu_q, cu_k, mq, mk, sink,
                                       p.softmax_scale, p.causal, window(p),
                                       deterministic=deterministic, dropout=dropout)
    torch.cuda.synchronize()
    return out, lse, dq, dk, dv, ds


def run_decode(d, num_splits=0, k_dev=None, v_dev=None):
    td = tdtype(d)
    q = dev(d.q, td)
    k = k_dev if k_dev is not None else dev(d.k, td)
    v = v_dev if v_dev is not None else dev(d.v, td)
    cu_k = dev(d.cu_seqlens_k)
    sink = None if d.sink is None else dev(d.sink)
    mk = max(int(np.diff(d.cu_seqlens_k).max()), 1)
    out, lse = sab.attn_sink_decode(q, k, v, cu_k, mk, sink, d.softmax_scale, d.causal,
                                    (d.window_left, d.window_right), num_splits)
    torch.cuda.synchronize()
    return out, lse
