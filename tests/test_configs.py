"""The five workload configurations at full size, in the launch configuration bench.py
times.  Small configs are compared element by element; large ones on sampled rows
(and, for the backward, whole (sequence, head) groups plus every dsink value),
each sample computed by the oracle one by one."""

import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_grad, check_lse, check_out, to_np
from _oracle_pool import dsink_term, group_bwd, pool_map

pytestmark = pytest.mark.gpu

try:
    import torch
    from gpu_util import dev, run_decode, run_fwd
    import softmax_attn_sink_b200 as sab
except Exception:
    pass


def _sample_rows(L, rng, extra=8):
    fixed = [0, 1, 2, 63, 64, 127, 128, 129, L // 2, L - 2, L - 1]
    rows = sorted(set([r for r in fixed if 0 <= r < L] + list(rng.integers(0, L, size=extra))))
    return rows


@pytest.mark.parametrize("causal", [False, True])
def test_config1_fixed_256_d64(causal):
    p = W.config1(causal)
    out, lse = run_fwd(p)
    ro, rl = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, causal)
    check_out(to_np(out), ro, "bf16")
    check_lse(to_np(lse), rl, "bf16")


def test_config2_varlen_gqa_causal_sampled():
    p = W.config2()
    out, lse = run_fwd(p)
    o, l = to_np(out), to_np(lse)
    rng = np.random.default_rng(100)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, -1, -1)
    for b in range(16):
        q0, q1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
        for h in rng.choice(32, size=3, replace=False):
            rows = _sample_rows(q1 - q0, rng)
            ro, rl = ref.fwd_rows(p.q, p.k, p.v, *a, b=b, h=int(h), rows=rows)
            idx = np.asarray(rows) + q0
            check_out(o[idx, h], ro, "bf16", f"out[b={b},h={h}]")
            check_lse(l[h, idx], rl, "bf16", f"lse[b={b},h={h}]")


def test_config3_training_fwd_bwd_sampled():
    p = W.config3()
    td = torch.bfloat16
    q, k, v, do = dev(p.q, td), dev(p.k, td), dev(p.v, td), dev(p.dout, td)
    cu = dev(p.cu_seqlens_q)
    sink = dev(p.sink)
    out, lse = sab.attn_sink_fwd(q, k, v, cu, cu, 8192, 8192, sink, p.softmax_scale, True)
    dq, dk, dv, ds = sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, 8192, 8192, sink,
                                       p.softmax_scale, True)
    torch.cuda.synchronize()
    o, l = to_np(out), to_np(lse)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, -1, -1)
    rng = np.random.default_rng(101)
    for b in range(4):
        for h in (0, 7, 15):
            rows = _sample_rows(8192, rng)
            ro, rl = ref.fwd_rows(p.q, p.k, p.v, *a, b=b, h=h, rows=rows)
            idx = np.asarray(rows) + 8192 * b
            check_out(o[idx, h], ro, "bf16", f"out[b={b},h={h}]")
            check_lse(l[h, idx], rl, "bf16", f"lse[b={b},h={h}]")
    # The backward runs the (sequence, kv head) groups in bands of 8 (four sequences x 16
    # heads = 64 groups; each band is one sequence's heads 0-7 or 8-15): dq / dk / dv of
    # every band's first group, and all 16 dsink values, each a sum over the four sequences.
    firsts = [(b, g) for b in range(4) for g in (0, 8)]
    sl = lambda b: slice(8192 * b, 8192 * (b + 1))  # noqa: E731
    gitems = [(p.q[sl(b), g:g + 1], p.k[sl(b), g:g + 1], p.v[sl(b), g:g + 1], p.dout[sl(b), g:g + 1],
               p.sink[g:g + 1], p.softmax_scale, True, -1, -1) for b, g in firsts]
    ditems = [(p.q[sl(b), h], p.k[sl(b), h], p.v[sl(b), h], p.dout[sl(b), h], float(p.sink[h]),
               p.softmax_scale, True, -1, -1) for b in range(4) for h in range(16) if (b, h) not in firsts]
    dkeys = [(b, h) for b in range(4) for h in range(16) if (b, h) not in firsts]
    gres = pool_map(group_bwd, gitems)
    dres = pool_map(dsink_term, ditems)
    gdq, gdk, gdv = to_np(dq), to_np(dk), to_np(dv)
    total = np.zeros(16)
    for (b, g), (rq, rk, rv, rs) in zip(firsts, gres):
        check_grad(gdq[sl(b), g], rq[:, 0], "bf16", f"dq[b={b},h={g}]")
        check_grad(gdk[sl(b), g], rk, "bf16", f"dk[b={b},g={g}]")
        check_grad(gdv[sl(b), g], rv, "bf16", f"dv[b={b},g={g}]")
        total[g] += rs[0]
    for (b, h), t in zip(dkeys, dres):
        total[h] += t
    print("dsink gpu   ", np.array2string(to_np(ds), precision=5, max_line_width=200))
    print("dsink oracle", np.array2string(total, precision=5, max_line_width=200))
    check_grad(to_np(ds), total, "bf16", "dsink")


def test_config3_training_with_dropout_sampled():
    """The training workload with dropout p = 0.1 at full size: sampled forward rows and one
    whole (sequence, head) of the backward (dsink with dropout is checked on the small cases
    of test_dropout.py: its oracle needs every row's keep bytes of the head)."""
    p = W.config3()
    drop = (0.1, 0x5EED5EED1234ABCD, 3)
    td = torch.bfloat16
    q, k, v, do = dev(p.q, td), dev(p.k, td), dev(p.v, td), dev(p.dout, td)
    cu = dev(p.cu_seqlens_q)
    sink = dev(p.sink)
    out, lse = sab.attn_sink_fwd(q, k, v, cu, cu, 8192, 8192, sink, p.softmax_scale, True, dropout=drop)
    dq, dk, dv, ds = sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, 8192, 8192, sink,
                                       p.softmax_scale, True, dropout=drop)
    torch.cuda.synchronize()
    o, l = to_np(out), to_np(lse)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, -1, -1)
    rng = np.random.default_rng(102)
    for b in (0, 3):
        for h in (2, 11):
            rows = _sample_rows(8192, rng)
            ro, rl = ref.fwd_rows(p.q, p.k, p.v, *a, b=b, h=h, rows=rows, dropout=drop)
            idx = np.asarray(rows) + 8192 * b
            check_out(o[idx, h], ro, "bf16", f"out[b={b},h={h}]")
            check_lse(l[h, idx], rl, "bf16", f"lse[b={b},h={h}]")
    b, g = 2, 9
    gq, gk, gv, gs = ref.bwd_sequence_group(p.q, p.k, p.v, p.dout, *a, b=b, g=g, dropout=drop)
    sl = slice(8192 * b, 8192 * (b + 1))
    check_grad(to_np(dq[sl, g]), gq[:, 0], "bf16", "dq")
    check_grad(to_np(dk[sl, g]), gk, "bf16", "dk")
    check_grad(to_np(dv[sl, g]), gv, "bf16", "dv")


@pytest.mark.parametrize("n", [1.0, 0.5, 3.0])
def test_config4_softmax_n_window(n):
    p = W.config4(n)
    out, lse = run_fwd(p)
    ro, rl = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                     True, 512, 0)
    check_out(to_np(out), ro, "bf16")
    check_lse(to_np(lse), rl, "bf16")


def test_config5_decode_sampled():
    d = W.config5_meta()
    total_k = int(d.cu_seqlens_k[-1])
    k, v = W.decode_kv_on_device(total_k, 8, 128, 128, seed=4)
    out, lse = run_decode(d, 0, k, v)
    o, l = to_np(out), to_np(lse)
    rng = np.random.default_rng(102)
    for b in sorted(set([0, 63] + list(rng.integers(0, 64, size=4)))):
        k0, k1 = int(d.cu_seqlens_k[b]), int(d.cu_seqlens_k[b + 1])
        for g in (0, int(rng.integers(1, 8))):
            kh = k[k0:k1, g].float().cpu().numpy()[:, None, :]
            vh = v[k0:k1, g].float().cpu().numpy()[:, None, :]
            heads = list(range(g * 8, g * 8 + 8))
            qq = d.q[b:b + 1, heads]
            ro, rl = ref.decode(qq, kh, vh, np.array([0, k1 - k0]), d.sink[heads], d.softmax_scale)
            check_out(o[b, heads], ro[0], "bf16", f"out[b={b},g={g}]")
            check_lse(l[heads, b], rl[:, 0], "bf16", f"lse[b={b},g={g}]")
