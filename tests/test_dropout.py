"""Dropout on the sink-normalised probabilities: the CUDA forward and backward against the
oracle's fwd / bwd with the same (p, seed, offset).

Two kinds of check.  On random inputs, every output element (and the gradients' relative
L2 error) is compared with the oracle.  On structured inputs (q = 0 so every visible key
has the same probability, sink = -inf, one-hot values or output gradients, windows of at
most 128 keys) each kept or dropped decision shows up as one nonzero or zero output
element, so the keep mask the kernels drew is compared with the oracle's bit for bit: a
wrong counter word, byte, row or head index cannot hide under a tolerance."""
import zlib

import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_grad, check_lse, check_out, to_np

pytestmark = pytest.mark.gpu

try:
    from gpu_util import run_bwd, run_fwd
except Exception:  # torch without CUDA still imports; the calls fail at run time
    pass

BIG_SEED = 0x9E3779B97F4A7C15   # both key words nonzero


def _seed(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


_LENS_P = [int(n) for n in np.random.default_rng(41).integers(0, 600, size=24)] + [0, 1]
_LENS_G = [int(n) for n in np.random.default_rng(42).integers(0, 5, size=9000)]

FWD_CASES = [
    # name, lens_q, lens_k, hq, hkv, dk, dv, causal, wl, wr, sink, dtype, p
    ("causal_gqa_p10", [300, 129, 0, 257], [300, 129, 0, 257], 8, 2, 128, 128, True, -1, -1,
     "normal", "bf16", 0.1),
    ("full_sq_ne_sk_dv64_p30", [200, 3, 333], [260, 300, 100], 4, 4, 128, 64, False, -1, -1,
     "uniform", "bf16", 0.3),
    ("window_p50", [400, 257], [400, 300], 4, 1, 128, 128, True, 64, 0, "normal", "bf16", 0.5),
    ("dk64_dv64_p20", [257, 64], [257, 64], 4, 2, 64, 64, False, -1, -1, "normal", "bf16", 0.2),
    ("dk64_dv128_odd_group_p10", [300, 129], [333, 200], 3, 1, 64, 128, True, 100, 0, "normal",
     "bf16", 0.1),
    ("fp16_causal_gqa_p10", [300, 129, 0, 257], [300, 129, 0, 257], 8, 2, 128, 128, True, -1, -1,
     "normal", "fp16", 0.1),
    ("fp16_neg_inf_sink_p25", [5, 260], [2, 260], 4, 2, 128, 128, True, -1, -1, "neg_inf", "fp16",
     0.25),
    ("persistent_many_items_p15", _LENS_P, _LENS_P, 6, 2, 128, 128, True, -1, -1, "normal", "bf16",
     0.15),
    ("grid_mode_p10", _LENS_G, _LENS_G, 2, 1, 128, 128, True, -1, -1, "normal", "bf16", 0.1),
    ("dk64_dv32_window_p10", [300, 129], [333, 200], 2, 1, 64, 32, True, 100, 0, "normal", "bf16", 0.1),
    ("d256_causal_gqa_p20", [300, 129, 0, 257], [300, 129, 0, 257], 4, 2, 256, 256, True, -1, -1,
     "normal", "bf16", 0.2),
    ("d256_fp16_window_p10", [200, 65], [230, 90], 2, 1, 256, 256, True, 70, 0, "normal", "fp16", 0.1),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fwd_dropout_matches_oracle(case):
    name, lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype, pdrop = case
    p = W.random_problem(_seed(name), lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype)
    drop = (pdrop, BIG_SEED + _seed(name), _seed(name) * 7)
    out, lse = run_fwd(p, drop)
    ro, rl = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                     p.causal, p.window_left, p.window_right, dropout=drop)
    check_out(to_np(out), ro, dtype)
    check_lse(to_np(lse), rl, dtype)


BWD_CASES = [
    # name, lens_q, lens_k, hq, hkv, dv, causal, wl, wr, sink, dtype, p
    ("causal_gqa_p10", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 128, True, -1, -1, "normal",
     "bf16", 0.1),
    ("dv64_window_p30", [260], [300], 2, 1, 64, True, 50, 0, "normal", "bf16", 0.3),
    ("full_sq_ne_sk_p20", [5, 130], [2, 200], 4, 2, 128, False, -1, -1, "uniform", "bf16", 0.2),
    ("long_gqa4_p10", [700, 300], [700, 300], 8, 2, 128, True, 200, 0, "normal", "bf16", 0.1),
    ("fp16_causal_p50", [300, 200], [300, 200], 4, 4, 128, True, -1, -1, "normal", "fp16", 0.5),
    ("fp16_dv64_p10", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 64, True, -1, -1, "normal", "fp16",
     0.1),
]


BWD_CASES += [
    # head dim 256 (dk = dv = 256): the dQ / dK / dV kernels with dropout
    ("d256_causal_gqa_p10", [1, 129, 0, 257], [1, 129, 0, 257], 4, 2, 256, True, -1, -1, "normal",
     "bf16", 0.1),
    ("d256_fp16_window_sq_ne_sk_p30", [200, 5], [230, 90], 2, 1, 256, True, 70, 0, "normal", "fp16", 0.3),
    # head dim 64 (the dv field reads "64x<dv>"): the d = 64 dK/dV kernel with dropout
    ("dk64_dv64_causal_gqa_p20", [1, 129, 0, 257], [1, 129, 0, 257], 4, 2, "64x64", True, -1, -1,
     "normal", "bf16", 0.2),
    ("dk64_dv32_causal_p20", [1, 129, 0, 257], [1, 129, 0, 257], 4, 2, "64x32", True, -1, -1,
     "normal", "bf16", 0.2),
    ("dk128_dv32_window_p10", [300, 70], [333, 90], 2, 1, "128x32", True, 100, 0, "normal", "bf16", 0.1),
    ("dk64_dv128_fp16_window_p10", [300, 70], [333, 90], 4, 1, "64x128", True, 100, 0, "uniform", "fp16",
     0.1),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_dropout_matches_oracle(case):
    name, lq, lk, hq, hkv, dv, causal, wl, wr, sink, dtype, pdrop = case
    if isinstance(dv, str):
        dk, dv = (int(x) for x in dv.split("x"))
    else:
        dk = 256 if dv == 256 else 128
    p = W.random_problem(_seed(name) + 5, lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype,
                         with_dout=True)
    drop = (pdrop, BIG_SEED ^ _seed(name), 3 + _seed(name))
    out, lse, dq, dk, dv_, ds = run_bwd(p, dropout=drop)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, p.causal, wl, wr)
    ro, _ = ref.fwd(p.q, p.k, p.v, *a, dropout=drop)
    check_out(to_np(out), ro, dtype)
    rdq, rdk, rdv, rds = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=drop)
    check_grad(to_np(dq), rdq, dtype, "dq")
    check_grad(to_np(dk), rdk, dtype, "dk")
    check_grad(to_np(dv_), rdv, dtype, "dv")
    if p.sink is not None:
        check_grad(to_np(ds), rds, dtype, "dsink")


# --- the keep mask, bit for bit -----------------------------------------------------------

def _visible_pairs(p):
    """Per (sequence, q head): packed row offset, key offset, visible mask [sq, sk]."""
    for b in range(p.batch):
        q0, q1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
        k0, k1 = int(p.cu_seqlens_k[b]), int(p.cu_seqlens_k[b + 1])
        vis = ref.allowed_mask(q1 - q0, k1 - k0, p.causal, p.window_left, p.window_right)
        yield b, q0, q1, k0, k1, vis


def _structured(lens_q, lens_k, hq, hkv, causal, wl, wr, dtype, for_bwd, d=128):
    """q = 0 (every visible key equally likely), sink = -inf, head dim d.  Forward: v one-hot
    on key position mod d, so out[i, h, j % d] = P Z for the one visible key j there.
    Backward: k one-hot on key position, v = 1, dout one-hot on query position, so
    dv[j, :, i % d] collects P Z of row i and dq[i, h, j % d] = scale dS_ij."""
    cu_q, cu_k = W.cu_from_lengths(lens_q), W.cu_from_lengths(lens_k)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = np.zeros((tq, hq, d), np.float32)
    k = np.zeros((tk, hkv, d), np.float32)
    v = np.zeros((tk, hkv, d), np.float32)
    dout = np.zeros((tq, hq, d), np.float32) if for_bwd else None
    for b in range(len(lens_q)):
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        pos = np.arange(k1 - k0)
        if for_bwd:
            k[k0 + pos, :, pos % d] = 1.0
            v[k0:k1] = 1.0
            q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
            qp = np.arange(q1 - q0)
            dout[q0 + qp, :, qp % d] = 1.0
        else:
            v[k0 + pos, :, pos % d] = 1.0
    sink = np.full(hq, -np.inf, np.float32)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    return W.Problem(q, k, v, cu_q, cu_k, sink, scale, causal, wl, wr, dtype, dout, "structured")


MASK_CASES = [
    # name, lens_q, lens_k, hq, hkv, causal, wl, wr, dtype, p (head dim 128)
    ("two_sided_gqa_p10", [300, 517, 129, 0, 1], [300, 517, 129, 0, 1], 4, 2, False, 60, 60, "bf16",
     0.1),
    ("causal_sk_gt_sq_p50", [260, 190], [297, 400], 2, 1, True, 127, 0, "bf16", 0.5),
    ("causal_mha_p90", [385, 128], [385, 128], 3, 3, True, 100, 0, "fp16", 0.9),
    # 256 (1 - p) = 230.5 exactly: T = 231 on both sides (halves round up)
    ("half_way_threshold", [200], [200], 2, 2, False, 50, 50, "bf16", 25.5 / 256),
]


@pytest.mark.parametrize("case,d", [(c, 128) for c in MASK_CASES] + [
    (("d256_two_sided_p30", [300, 517], [300, 517], 2, 1, False, 120, 120, "bf16", 0.3), 256)],
    ids=[c[0] for c in MASK_CASES] + ["d256_two_sided_p30"])
def test_fwd_dropout_keep_mask_is_exact(case, d):
    name, lq, lk, hq, hkv, causal, wl, wr, dtype, pdrop = case
    p = _structured(lq, lk, hq, hkv, causal, wl, wr, dtype, for_bwd=False, d=d)
    drop = (pdrop, BIG_SEED + _seed(name), 11)
    t = ref.dropout_threshold(pdrop)
    want = np.zeros((int(p.cu_seqlens_q[-1]), hq, d), bool)
    for b, q0, q1, k0, k1, vis in _visible_pairs(p):
        cols = np.arange(k1 - k0) % d
        for i in range(q1 - q0):   # a row sees at most d consecutive keys: one per column
            assert len(set(cols[vis[i]])) == int(vis[i].sum())
        for h in range(hq):
            keep = ref.dropout_keep(drop[1], drop[2], t, np.arange(q0, q1), h, k1 - k0) & vis
            for i, j in zip(*np.nonzero(keep)):
                want[q0 + i, h, cols[j]] = True
    out, _ = run_fwd(p, drop)
    got = to_np(out) != 0.0
    assert want.any() and not want.all()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} keep decisions differ; first (row, head, col) {bad[:5].tolist()}"


@pytest.mark.parametrize("case,d", [(c, 128) for c in MASK_CASES[:2]] + [
    (("causal_fp16_dv_p30", [333, 129], [333, 140], 4, 2, True, 90, 0, "fp16", 0.3), 128),
    (("d256_two_sided_gqa_p20", [300, 517], [300, 517], 4, 2, False, 120, 120, "bf16", 0.2), 256),
    (("d64_causal_gqa_p25", [300, 200], [300, 200], 4, 2, True, 63, 0, "bf16", 0.25), 64)],
    ids=[c[0] for c in MASK_CASES[:2]] + ["causal_fp16_dv_p30", "d256_two_sided_gqa_p20", "d64_causal_gqa_p25"])
def test_bwd_dropout_keep_mask_is_exact(case, d):
    """dv carries the keep mask bit for bit; dq, the difference of kept and dropped terms,
    is checked element-wise within a tenth of the gap between the two."""
    name, lq, lk, hq, hkv, causal, wl, wr, dtype, pdrop = case
    p = _structured(lq, lk, hq, hkv, causal, wl, wr, dtype, for_bwd=True, d=d)
    drop = (pdrop, BIG_SEED ^ (_seed(name) << 40), 5)
    t = ref.dropout_threshold(pdrop)
    grp = hq // hkv
    want_dv = np.zeros((int(p.cu_seqlens_k[-1]), hkv, d), bool)
    gap = np.zeros((int(p.cu_seqlens_q[-1]), hq, 1))
    for b, q0, q1, k0, k1, vis in _visible_pairs(p):
        rows = np.arange(q1 - q0) % d
        for j in range(k1 - k0):   # a key is seen by at most d consecutive rows
            assert len(set(rows[vis[:, j]])) == int(vis[:, j].sum())
        n = np.maximum(vis.sum(axis=1), 1)
        for h in range(hq):
            keep = ref.dropout_keep(drop[1], drop[2], t, np.arange(q0, q1), h, k1 - k0) & vis
            for i, j in zip(*np.nonzero(keep)):
                want_dv[k0 + j, h // grp, rows[i]] = True
            gap[q0:q1, h, 0] = p.softmax_scale * (256.0 / t) / n
    out, lse, dq, dk, dv, ds = run_bwd(p, dropout=drop)
    got_dv = to_np(dv) != 0.0
    assert want_dv.any() and not want_dv.all()
    bad = np.argwhere(got_dv != want_dv)
    assert bad.size == 0, f"{len(bad)} keep decisions differ in dv; first {bad[:5].tolist()}"
    assert np.all(to_np(dk) == 0.0)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, p.causal, wl, wr)
    rdq, _, _, _ = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=drop)
    err = np.abs(to_np(dq) - rdq)
    assert np.all(err <= 0.1 * gap), f"dq: max err / gap {float((err / gap).max()):.3f}"


# --- identities ---------------------------------------------------------------------------

def test_dropout_repeats_for_equal_seed_and_offset_and_changes_otherwise():
    p = W.random_problem(61, [300, 257], [300, 257], 4, 2, 128, 128, True, with_dout=True)
    base = (0.2, BIG_SEED, 9)
    o1, l1, dq1, dk1, dv1, ds1 = run_bwd(p, dropout=base)
    o2, l2, dq2, dk2, dv2, ds2 = run_bwd(p, dropout=base)
    for x, y in ((o1, o2), (l1, l2), (dq1, dq2), (dk1, dk2), (dv1, dv2), (ds1, ds2)):
        assert np.array_equal(to_np(x), to_np(y))
    o3, l3 = run_fwd(p, (0.2, BIG_SEED, 10))           # next offset: a fresh mask
    o4, _ = run_fwd(p, (0.2, BIG_SEED ^ (1 << 63), 9))  # high key word changed
    o5, _ = run_fwd(p, (0.2, BIG_SEED ^ 1, 9))          # low key word changed
    for o in (o3, o4, o5):
        assert not np.array_equal(to_np(o), to_np(o1))
    assert np.array_equal(to_np(l3), to_np(l1))         # lse does not see the mask


def test_dropout_with_p_zero_matches_no_dropout():
    """p = 0 keeps every element with weight 1: the forward and backward agree with the
    plain (deterministic) path within the kernels' tolerance."""
    p = W.random_problem(62, [300, 129], [300, 129], 4, 2, 128, 128, True, with_dout=True)
    plain = run_bwd(p, deterministic=True)
    drop = run_bwd(p, dropout=(0.0, BIG_SEED, 0))
    check_out(to_np(drop[0]), to_np(plain[0]), "bf16")
    check_lse(to_np(drop[1]), to_np(plain[1]), "bf16")
    for idx, name in ((2, "dq"), (3, "dk"), (4, "dv"), (5, "dsink")):
        check_grad(to_np(drop[idx]), to_np(plain[idx]), "bf16", name)
