"""Pins for the fp64 oracle: each check ties the oracle to something other than itself
(an identity the pages state, a library routine, a closed form, brute force, or
finite differences), chosen so that a dropped term, a wrong sign or index, or a
transposed operand in ``oracle/ref.py`` fails at least one of them.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import ref
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_masks():
    cases = []
    name, rows, hdr = None, [], None
    with open(os.path.join(GOLDEN, "bottom_right_masks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                if name:
                    cases.append((name, hdr, np.array(rows, dtype=bool)))
                parts = line.strip("[]").split()
                name, hdr, rows = parts[0], tuple(int(x) for x in parts[1:]), []
            else:
                rows.append([int(x) for x in line.split()])
    if name:
        cases.append((name, hdr, np.array(rows, dtype=bool)))
    return cases


MASKS = _load_masks()


# --- P4: bottom-right masks ------------------------------------------------------------

@pytest.mark.parametrize("name,hdr,expect", MASKS, ids=[c[0] for c in MASKS])
def test_p4_bottom_right_masks(name, hdr, expect):
    sq, sk, causal, wl, wr = hdr
    assert expect.shape == (sq, sk)
    got = ref.allowed_mask(sq, sk, bool(causal), wl, wr)
    np.testing.assert_array_equal(got, expect)


def test_golden_file_has_the_issue_cases():
    names = {c[0] for c in MASKS}
    assert {"q2_k5", "q5_k2", "q1_k5"} <= names


# --- brute force with scalar loops on tiny inputs ------------------------------------

def _brute_force(p):
    """Scalar-loop sink attention: every pair, every dimension, math.exp only."""
    hq, hkv = p.q.shape[1], p.k.shape[1]
    dv = p.v.shape[2]
    out = np.zeros((p.q.shape[0], hq, dv))
    lse = np.full((hq, p.q.shape[0]), -np.inf)
    for b in range(len(p.cu_seqlens_q) - 1):
        q0, q1 = int(p.cu_seqlens_q[b]), int(p.cu_seqlens_q[b + 1])
        k0, k1 = int(p.cu_seqlens_k[b]), int(p.cu_seqlens_k[b + 1])
        sq, sk = q1 - q0, k1 - k0
        for h in range(hq):
            g = h * hkv // hq
            sink = -math.inf if p.sink is None else float(p.sink[h])
            for i in range(sq):
                scores = []
                for j in range(sk):
                    pos = i + sk - sq
                    ok = j <= pos if p.causal else True
                    if p.window_right >= 0:
                        ok = ok and j <= pos + p.window_right
                    if p.window_left >= 0:
                        ok = ok and j >= pos - p.window_left
                    if ok:
                        s = sum(float(p.q[q0 + i, h, c]) * float(p.k[k0 + j, g, c])
                                for c in range(p.q.shape[2])) * p.softmax_scale
                        scores.append((j, s))
                if scores:
                    mx = max(s for _, s in scores)
                    lse[h, q0 + i] = mx + math.log(sum(math.exp(s - mx) for _, s in scores))
                m = max([sink] + [s for _, s in scores])
                if m == -math.inf:
                    continue
                den = sum(math.exp(s - m) for _, s in scores) + math.exp(sink - m)
                for c in range(dv):
                    out[q0 + i, h, c] = sum(math.exp(s - m) * float(p.v[k0 + j, g, c])
                                            for j, s in scores) / den
    return out, lse


@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (True, 2, -1),
                                          (False, 1, 2), (False, -1, 0)])
def test_oracle_matches_scalar_brute_force(causal, wl, wr):
    p = W.random_problem(11, [3, 0, 5, 2], [4, 2, 5, 6], hq=4, hkv=2, dk=5, dv=3,
                         causal=causal, window_left=wl, window_right=wr, dtype="fp32",
                         softmax_scale=0.37)
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                       causal, wl, wr)
    bo, bl = _brute_force(p)
    np.testing.assert_allclose(out, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(np.isinf(lse), np.isinf(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=1e-12, atol=1e-13)


# --- P1: appended-column softmax == sigmoid-scaled softmax == oracle -------------------

def test_p1_appended_sink_column_identity():
    p = W.random_problem(1, [7], [9], hq=2, hkv=2, dk=6, dv=4, dtype="fp32", softmax_scale=0.41)
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale)
    for h in range(2):
        q = torch.tensor(p.q[:, h], dtype=torch.float64)
        k = torch.tensor(p.k[:, h], dtype=torch.float64)
        v = torch.tensor(p.v[:, h], dtype=torch.float64)
        S = (q @ k.T) * p.softmax_scale
        off = float(p.sink[h])
        # (a) softmax over [S, offset], drop the appended column
        Pa = torch.softmax(torch.cat([S, torch.full((S.shape[0], 1), off, dtype=torch.float64)], 1), 1)[:, :-1]
        # (b) softmax(S) * sigmoid(logsumexp(S) - offset)
        Pb = torch.softmax(S, 1) * torch.sigmoid(torch.logsumexp(S, 1) - off)[:, None]
        np.testing.assert_allclose(Pa.numpy(), Pb.numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out[:, h], (Pa @ v).numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[h], torch.logsumexp(S, 1).numpy(), rtol=1e-12)
        r = ref.attend_head(p.q[:, h], p.k[:, h], p.v[:, h], off, p.softmax_scale,
                            ref.allowed_mask(7, 9, False))
        np.testing.assert_allclose(r["P"], Pa.numpy(), rtol=1e-12, atol=1e-14)


# --- P2: softmax_n == sink = log n -------------------------------------------------------

@pytest.mark.parametrize("n", [1.0, 0.5, 3.0])
def test_p2_softmax_n_is_sink_log_n(n):
    p = W.random_problem(2, [5], [8], hq=1, hkv=1, dk=4, dv=3, dtype="fp32", softmax_scale=0.5,
                         sink=math.log(n))
    out, _ = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale)
    x = p.softmax_scale * (p.q[:, 0].astype(np.float64) @ p.k[:, 0].astype(np.float64).T)
    ex = np.exp(x)                                  # no max subtraction: small inputs
    n_fp32 = math.exp(float(p.sink[0]))             # the sink is handed over as fp32
    assert abs(n_fp32 - n) <= 1e-7 * n
    probs = ex / (n_fp32 + ex.sum(axis=1, keepdims=True))
    np.testing.assert_allclose(out[:, 0], probs @ p.v[:, 0].astype(np.float64), rtol=1e-12)


def test_p2_sink_is_not_multiplied_by_scale():
    # with scale != 1, a sink read in pre-scale units would give a different denominator
    n = 3.0
    p = W.random_problem(3, [4], [6], hq=1, hkv=1, dk=4, dv=2, dtype="fp32", softmax_scale=0.25,
                         sink=math.log(n))
    out, _ = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale)
    x = 0.25 * (p.q[:, 0].astype(np.float64) @ p.k[:, 0].astype(np.float64).T)
    wrong = np.exp(x) / (n ** 0.25 + np.exp(x).sum(1, keepdims=True)) @ p.v[:, 0]
    assert np.abs(out[:, 0] - wrong).max() > 1e-3


# --- P3: sink = -inf is vanilla softmax attention (library cross-check) ---------------

@pytest.mark.parametrize("causal,sq,sk", [(False, 6, 9), (True, 6, 9), (True, 7, 7)])
def test_p3_neg_inf_sink_is_sdpa(causal, sq, sk):
    p = W.random_problem(4, [sq], [sk], hq=4, hkv=2, dk=8, dv=5, causal=causal, dtype="fp32",
                         sink="neg_inf")
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                       causal)
    out2, lse2 = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, None, p.softmax_scale,
                         causal)
    np.testing.assert_array_equal(out, out2)
    # explicit bottom-right mask built independently: key j visible iff j - i <= sk - sq
    i = torch.arange(sq)[:, None]
    j = torch.arange(sk)[None, :]
    mask = (j - i <= sk - sq) if causal else torch.ones(sq, sk, dtype=torch.bool)
    for h in range(4):
        q = torch.tensor(p.q[:, h], dtype=torch.float64)[None, None]
        k = torch.tensor(p.k[:, h // 2], dtype=torch.float64)[None, None]
        v = torch.tensor(p.v[:, h // 2], dtype=torch.float64)[None, None]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                             scale=p.softmax_scale)
        np.testing.assert_allclose(out[:, h], o[0, 0].numpy(), rtol=1e-11, atol=1e-12)
        S = (q[0, 0] @ k[0, 0].T) * p.softmax_scale
        np.testing.assert_allclose(lse[h], torch.logsumexp(S.masked_fill(~mask, -math.inf), 1).numpy(),
                                   rtol=1e-12)


# --- P5: fully masked rows ------------------------------------------------------------

@pytest.mark.parametrize("sink", ["normal", "neg_inf"])
def test_p5_fully_masked_rows(sink):
    # q=5, k=2 causal: rows 0-2 see nothing; second sequence has sk = 0
    p = W.random_problem(5, [5, 3], [2, 0], hq=2, hkv=1, dk=4, dv=3, causal=True, dtype="fp32",
                         sink=sink, with_dout=True)
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    dead = [0, 1, 2, 5, 6, 7]
    assert np.all(out[dead] == 0.0)
    assert np.all(np.isneginf(lse[:, dead]))
    assert np.all(np.isfinite(out))
    dq, dk, dv, ds = ref.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens_q, p.cu_seqlens_k, p.sink,
                             p.softmax_scale, True)
    assert np.all(dq[dead] == 0.0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv)) and np.all(np.isfinite(ds))
    # dead rows add nothing: dropping them leaves dk, dv and dsink unchanged
    keep = [3, 4]
    cu_q = np.array([0, 2], dtype=np.int32)
    cu_k = np.array([0, 2], dtype=np.int32)
    dq2, dk2, dv2, ds2 = ref.bwd(p.q[keep], p.k, p.v, p.dout[keep], cu_q, cu_k, p.sink,
                                 p.softmax_scale, True)
    np.testing.assert_allclose(dk, dk2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(dv, dv2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(ds, ds2, rtol=1e-13, atol=1e-15)


# --- P6: closed form with q = 0 -------------------------------------------------------

@pytest.mark.parametrize("sink", [-1.3, 0.0, 2.5])
def test_p6_zero_query_closed_form(sink):
    p = W.random_problem(6, [4], [7], hq=1, hkv=1, dk=3, dv=5, causal=True, dtype="fp32",
                         sink=sink)
    q = np.zeros_like(p.q)
    out, lse = ref.fwd(q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    for i in range(4):
        L = i + 3 + 1                      # bottom-right: row i sees keys 0 .. i + 3
        expect = p.v[:L, 0].astype(np.float64).sum(0) / (L + math.exp(float(p.sink[0])))
        np.testing.assert_allclose(out[i, 0], expect, rtol=1e-13)
        assert abs(lse[0, i] - math.log(L)) < 1e-13


# --- P7: limits -----------------------------------------------------------------------

def test_p7_large_sink_limit():
    p = W.random_problem(7, [3], [5], hq=1, hkv=1, dk=4, dv=2, dtype="fp32", sink=60.0,
                         with_dout=True)
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale)
    assert np.abs(out).max() < 1e-20
    _, _, _, ds = ref.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens_q, p.cu_seqlens_k, p.sink,
                          p.softmax_scale)
    assert abs(ds[0]) < 1e-20
    # lse does not see the sink
    _, lse0 = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, None, p.softmax_scale)
    np.testing.assert_allclose(lse, lse0, rtol=1e-14)


# --- P8: probabilities plus the sink's share sum to one --------------------------------

def test_p8_rows_sum_to_one():
    p = W.random_problem(8, [6], [6], hq=1, hkv=1, dk=4, dv=2, causal=True, window_left=2,
                         dtype="fp32")
    r = ref.attend_head(p.q[:, 0], p.k[:, 0], p.v[:, 0], float(p.sink[0]), p.softmax_scale,
                        ref.allowed_mask(6, 6, True, 2, -1))
    np.testing.assert_allclose(r["P"].sum(1) + r["p_sink"], 1.0, rtol=1e-14)
    assert np.all(r["P"][~ref.allowed_mask(6, 6, True, 2, -1)] == 0)


# --- P9: finite differences -----------------------------------------------------------

def test_p9_gradients_match_finite_differences():
    p = W.random_problem(9, [3, 5], [4, 6], hq=4, hkv=2, dk=4, dv=3, causal=True,
                         window_left=3, dtype="fp32", with_dout=True)
    args = (p.cu_seqlens_q, p.cu_seqlens_k)
    q, k, v, do = (x.astype(np.float64) for x in (p.q, p.k, p.v, p.dout))
    sink = p.sink.astype(np.float64)

    def loss(q_, k_, v_, s_):
        o, _ = ref.fwd(q_, k_, v_, *args, s_, p.softmax_scale, True, 3, -1)
        return float((o * do).sum())

    dq, dk, dv, ds = ref.bwd(q, k, v, do, *args, sink, p.softmax_scale, True, 3, -1)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("sink", sink, ds)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = {"q": (xp, k, v, sink), "k": (q, xp, v, sink), "v": (q, k, xp, sink),
                 "sink": (q, k, v, xp)}[name]
            b = {"q": (xm, k, v, sink), "k": (q, xm, v, sink), "v": (q, k, xm, sink),
                 "sink": (q, k, v, xm)}[name]
            num[idx] = (loss(*a) - loss(*b)) / (2 * h)
        rel = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert rel <= 1e-6, (name, rel)


# --- P10: the backward in the form of the slime docstring -----------------------------------

def test_p10_learnable_offset_backward_form():
    p = W.random_problem(10, [9], [9], hq=2, hkv=1, dk=5, dv=4, dtype="fp32", with_dout=True,
                         sink=[0.3, -0.8])
    dq, dk, dv, ds = ref.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens_q, p.cu_seqlens_k, p.sink,
                             p.softmax_scale)
    dk_alt = np.zeros_like(dk)
    dv_alt = np.zeros_like(dv)
    for h in range(2):
        q = torch.tensor(p.q[:, h], dtype=torch.float64)
        k = torch.tensor(p.k[:, 0], dtype=torch.float64)
        v = torch.tensor(p.v[:, 0], dtype=torch.float64)
        do = torch.tensor(p.dout[:, h], dtype=torch.float64)
        S = (q @ k.T) * p.softmax_scale
        P_van = torch.softmax(S, 1)
        O_van = P_van @ v
        s = torch.sigmoid(torch.logsumexp(S, 1) - float(p.sink[h]))
        di = (do * O_van).sum(1)
        dP = do @ v.T
        dS = P_van * s[:, None] * (dP - (s * di)[:, None])
        np.testing.assert_allclose(dq[:, h], (p.softmax_scale * dS @ k).numpy(), rtol=1e-11, atol=1e-13)
        dk_alt[:, 0] += (p.softmax_scale * dS.T @ q).numpy()
        dv_alt[:, 0] += ((s[:, None] * P_van).T @ do).numpy()
        d_offset = -(di * s * (1 - s)).sum()
        np.testing.assert_allclose(ds[h], float(d_offset), rtol=1e-11)
    np.testing.assert_allclose(dk, dk_alt, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dv, dv_alt, rtol=1e-11, atol=1e-13)


# --- P11: structural invariances --------------------------------------------------------

def test_p11_varlen_equals_per_sequence():
    p = W.random_problem(12, [5, 1, 7], [6, 3, 7], hq=2, hkv=1, dk=4, dv=3, causal=True,
                         dtype="fp32")
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    for b in range(3):
        q0, q1 = p.cu_seqlens_q[b], p.cu_seqlens_q[b + 1]
        k0, k1 = p.cu_seqlens_k[b], p.cu_seqlens_k[b + 1]
        o1, l1 = ref.fwd(p.q[q0:q1], p.k[k0:k1], p.v[k0:k1], np.array([0, q1 - q0]),
                         np.array([0, k1 - k0]), p.sink, p.softmax_scale, True)
        np.testing.assert_allclose(out[q0:q1], o1, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(lse[:, q0:q1], l1, rtol=1e-14)


def test_p11_gqa_equals_repeated_kv():
    p = W.random_problem(13, [6], [8], hq=6, hkv=2, dk=4, dv=3, causal=True, dtype="fp32")
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    k_rep, v_rep = np.repeat(p.k, 3, axis=1), np.repeat(p.v, 3, axis=1)
    out2, lse2 = ref.fwd(p.q, k_rep, v_rep, p.cu_seqlens_q, p.cu_seqlens_k, p.sink,
                         p.softmax_scale, True)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_p11_key_permutation_invariance():
    p = W.random_problem(14, [5], [9], hq=2, hkv=2, dk=4, dv=3, dtype="fp32")
    out, lse = ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale)
    perm = np.random.default_rng(0).permutation(9)
    out2, lse2 = ref.fwd(p.q, p.k[perm], p.v[perm], p.cu_seqlens_q, p.cu_seqlens_k, p.sink,
                         p.softmax_scale)
    np.testing.assert_allclose(out, out2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, rtol=1e-13)


# --- P12: split-KV + LSE merge ----------------------------------------------------------

@pytest.mark.parametrize("splits", [1, 2, 3, 7, 40])
def test_p12_split_merge_equals_unsplit(splits):
    d = W.random_decode(15, [40, 17, 1], hq=4, hkv=2, dk=6, dv=5, causal=True, window_left=25)
    out, lse = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale, True, 25, -1)
    for b in range(3):
        k0, k1 = d.cu_seqlens_k[b], d.cu_seqlens_k[b + 1]
        row = ref.allowed_mask(1, k1 - k0, True, 25, -1)[0]
        for h in range(4):
            parts = ref.decode_partials(d.q[b, h], d.k[k0:k1, h // 2], d.v[k0:k1, h // 2],
                                        d.softmax_scale, row, splits)
            o, l = ref.merge_partials(parts, float(d.sink[h]))
            np.testing.assert_allclose(o, out[b, h], rtol=1e-12, atol=1e-14)
            assert abs(l - lse[h, b]) < 1e-12


def test_p12_sink_in_every_split_is_wrong():
    d = W.random_decode(16, [64], hq=1, hkv=1, dk=4, dv=3, sink=[0.7])
    out, _ = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale)
    row = ref.allowed_mask(1, 64, True)[0]
    parts = ref.decode_partials(d.q[0, 0], d.k[:, 0], d.v[:, 0], d.softmax_scale, row, 4)
    # planted mistake: normalise each split with its own sink term, then average by weight
    sink = 0.7
    num, den = 0.0, 0.0
    for m_c, l_c, o_c in parts:
        mm = max(m_c, sink)
        num = num + o_c * math.exp(m_c - mm) * 1.0
        den = den + l_c * math.exp(m_c - mm) + math.exp(sink - mm)
    wrong = num / den
    assert np.abs(wrong - out[0, 0]).max() > 1e-3


def test_decode_equals_fwd_with_one_query_per_sequence():
    d = W.random_decode(17, [5, 9], hq=2, hkv=1, dk=4, dv=4)
    out, lse = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale)
    # the decode example of PyTorch issue #108108 ("Benefits"): the one query sees every cached key
    for b, (k0, k1) in enumerate([(0, 5), (5, 14)]):
        for h in range(2):
            S = d.softmax_scale * (d.k[k0:k1, 0].astype(np.float64) @ d.q[b, h].astype(np.float64))
            np.testing.assert_allclose(lse[h, b], np.log(np.exp(S).sum()), rtol=1e-13)


# --- oracle helpers used by the parity tests ---------------------------------------------

def test_fwd_rows_and_group_bwd_match_full():
    p = W.random_problem(18, [7, 9], [7, 11], hq=4, hkv=2, dk=4, dv=3, causal=True,
                         window_left=4, dtype="fp32", with_dout=True)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, 4, -1)
    out, lse = ref.fwd(p.q, p.k, p.v, *a)
    o, l = ref.fwd_rows(p.q, p.k, p.v, *a, b=1, h=3, rows=[0, 4, 8])
    np.testing.assert_array_equal(o, out[[7, 11, 15], 3])
    np.testing.assert_array_equal(l, lse[3, [7, 11, 15]])
    dq, dk, dv, ds = ref.bwd(p.q, p.k, p.v, p.dout, *a)
    gq, gk, gv, gs = ref.bwd_sequence_group(p.q, p.k, p.v, p.dout, *a, b=1, g=1)
    np.testing.assert_allclose(gq, dq[7:16, 2:4], rtol=1e-14, atol=1e-15)
    # dk/dv of sequence 1 rows 7:18 only receive sequence-1 contributions
    np.testing.assert_allclose(gk, dk[7:18, 1], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(gv, dv[7:18, 1], rtol=1e-14, atol=1e-15)


def test_pair_count_matches_masks():
    cu_q = np.array([0, 3, 8])
    cu_k = np.array([0, 5, 7])
    n = ref.pair_count(cu_q, cu_k, 2, True, -1, -1)
    # seq 0: q3 k5 causal -> rows see 3,4,5 keys; seq 1: q5 k2 -> 0,0,0,1,2
    assert n == 2 * (3 + 4 + 5 + 1 + 2)


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(10000, dtype=np.float32) * 3
    ours = W.bf16_round(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours, theirs)


# --- P13: paged K/V (CANN flash_attn doc, "Paged Attention Parameter Group", PA_BBND) ----

def test_p13_paged_gather_literal():
    """Key t of a sequence is row t % block_size of block table[t // block_size]: a cache
    whose row r of block p holds (p, r), read through the table [2, 0] for 20 keys with
    block_size 16, gives (2, 0) ... (2, 15), then (0, 0) ... (0, 3)."""
    bs, nb = 16, 3
    cache = np.zeros((nb, bs, 1, 2))
    for p_ in range(nb):
        for r in range(bs):
            cache[p_, r, 0] = (p_, r)
    packed, cu = ref.gather_paged(cache, np.array([[2, 0, 1]], np.int32), np.array([20], np.int32), bs)
    expected = [(2, r) for r in range(16)] + [(0, r) for r in range(4)]
    assert cu.tolist() == [0, 20]
    assert packed[:, 0].tolist() == [list(map(float, e)) for e in expected]


def _scatter_to_cache(x, cu, table, bs, nb):
    """Write packed rows into a block cache, one key at a time, through the table."""
    cache = np.zeros((nb, bs) + x.shape[1:])
    for b in range(len(cu) - 1):
        for t in range(int(cu[b + 1] - cu[b])):
            cache[table[b][t // bs], t % bs] = x[cu[b] + t]
    return cache


@pytest.mark.parametrize("bs", [16, 48, 64])
def test_p13_paged_decode_equals_packed_decode(bs):
    """A cache filled through a random block table (physical blocks shuffled, tail blocks
    partly used, a zero-length sequence) decodes exactly like the packed keys."""
    rng = np.random.default_rng(130 + bs)
    lens = [37, 0, 130, 16, 95]
    p = W.random_problem(131 + bs, [1] * len(lens), lens, 4, 2, 16, 8, True, sink="normal")
    per = [-(-n // bs) for n in lens]
    max_blocks = max(per) + 1
    nb = sum(per) + 3
    perm = rng.permutation(nb)
    table = np.full((len(lens), max_blocks), nb - 1, np.int32)   # unused entries: any valid id
    i = 0
    for b, n in enumerate(per):
        table[b, :n] = perm[i:i + n]
        i += n
    kc = _scatter_to_cache(p.k, p.cu_seqlens_k, table, bs, nb)
    vc = _scatter_to_cache(p.v, p.cu_seqlens_k, table, bs, nb)
    used = np.array(lens, np.int32)
    o1, l1 = ref.decode_paged(p.q, kc, vc, table, used, bs, p.sink, p.softmax_scale, True)
    o2, l2 = ref.decode(p.q, p.k, p.v, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_p13_shared_prefix_block():
    """Two sequences whose tables name the same first block see the same first keys:
    with identical queries and one shared full block, their outputs agree."""
    bs = 16
    rng = np.random.default_rng(7)
    kc = W.bf16_round(rng.standard_normal((3, bs, 1, 8), dtype=np.float32))
    vc = W.bf16_round(rng.standard_normal((3, bs, 1, 8), dtype=np.float32))
    q = np.repeat(W.bf16_round(rng.standard_normal((1, 2, 8), dtype=np.float32)), 2, axis=0)
    table = np.array([[1, 2], [1, 0]], np.int32)
    o, l = ref.decode_paged(q, kc, vc, table, np.array([16, 16], np.int32), bs, None, 0.3, True)
    assert np.array_equal(o[0], o[1]) and np.array_equal(l[:, 0], l[:, 1])
    # and the result is attention over block 1 alone
    o_ref, _ = ref.decode(q[:1], kc[1], vc[1], np.array([0, 16]), None, 0.3, True)
    assert np.allclose(o[0], o_ref[0], rtol=0, atol=1e-15)


def test_fp16_rounding_matches_torch():
    """The fp16 inputs are the values torch's float16 conversion gives (nearest, ties to even)."""
    x = np.random.default_rng(3).standard_normal(10000).astype(np.float32) * 100
    x[:4] = [65504.0, 1e-8, -2.0 ** -24 * 1.5, 0.5 + 2.0 ** -12]
    assert np.array_equal(W.fp16_round(x), torch.from_numpy(x).to(torch.float16).float().numpy())


# --- P14: dropout (Philox4x32-10; slime wrapper's dropout_p) ------------------------------

def test_p14_philox_known_answers():
    """The oracle's Philox4x32-10 reproduces the published known-answer vectors."""
    path = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        got = [int(x) for x in ref.philox4x32_10(v[0:4], v[4:6])]
        assert got == v[6:10]


def test_p14_keep_rate_and_threshold():
    """Bytes below T are kept: over 2^18 decisions the kept share is T/256 within 4 sigma,
    and T = 256 keeps everything."""
    for p in (0.1, 0.5, 0.9):
        t = ref.dropout_threshold(p)
        keep = ref.dropout_keep(2024, 3, t, np.arange(256), 5, 1024)
        q = t / 256.0
        sigma = math.sqrt(q * (1 - q) / keep.size)
        assert abs(keep.mean() - q) < 4 * sigma
    assert ref.dropout_keep(1, 0, 256, np.arange(8), 0, 100).all()
    with pytest.raises(ValueError):
        ref.dropout_threshold(0.999)


def test_p14_threshold_rounds_halves_up_from_the_float_p():
    """T = floor(256 (1 - p) + 1/2) of the float32 p, exactly: 256 (1 - p) = 230.5 gives 231,
    0.5 gives 1, and a p whose float is just above a half-way point rounds down."""
    assert ref.dropout_threshold(25.5 / 256) == 231
    assert ref.dropout_threshold(1 - 0.5 / 256) == 1
    assert ref.dropout_threshold(0.75) == 64 and ref.dropout_threshold(0.0) == 256
    p = float(np.nextafter(np.float32(25.5 / 256), np.float32(1)))   # 256 (1 - p) just below 230.5
    assert ref.dropout_threshold(p) == 230


def test_p14_sampled_helpers_follow_fwd_and_bwd_with_dropout():
    """fwd_rows and bwd_sequence_group with dropout reproduce the rows and the (sequence, kv
    head) slice of fwd / bwd with the same dropout (the helpers used on full-size problems)."""
    p = W.random_problem(77, [40, 57], [50, 57], 4, 2, 8, 6, True, 20, 0, with_dout=True)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, 20, 0)
    drop = (0.3, 12345, 6)
    ro, rl = ref.fwd(p.q, p.k, p.v, *a, dropout=drop)
    rows = [0, 3, 17, 56]
    o, l = ref.fwd_rows(p.q, p.k, p.v, *a, b=1, h=3, rows=rows, dropout=drop)
    assert np.allclose(o, ro[40 + np.asarray(rows), 3], rtol=0, atol=1e-14)
    assert np.allclose(l, rl[3, 40 + np.asarray(rows)], rtol=0, atol=1e-14)
    dq, dk, dv, ds = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=drop)
    gq, gk, gv, gs = ref.bwd_sequence_group(p.q, p.k, p.v, p.dout, *a, b=1, g=1, dropout=drop)
    assert np.allclose(gq, dq[40:97, 2:4], atol=1e-13)
    assert np.allclose(gk, dk[50:107, 1], atol=1e-13) and np.allclose(gv, dv[50:107, 1], atol=1e-13)
    # dsink of a head sums its sequences: the slice's part plus sequence 0's
    g0 = ref.bwd_sequence_group(p.q, p.k, p.v, p.dout, *a, b=0, g=1, dropout=drop)[3]
    assert np.allclose(gs + g0, ds[2:4], atol=1e-13)


def test_p14_no_dropout_is_identity():
    """p = 0 (T = 256) gives exactly the forward and backward without dropout."""
    p = W.random_problem(140, [9, 5], [11, 5], 4, 2, 8, 6, True, dtype="fp32", with_dout=True)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    o1, l1 = ref.fwd(p.q, p.k, p.v, *a)
    o2, l2 = ref.fwd(p.q, p.k, p.v, *a, dropout=(0.0, 9, 1))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    g1 = ref.bwd(p.q, p.k, p.v, p.dout, *a)
    g2 = ref.bwd(p.q, p.k, p.v, p.dout, *a, dropout=(0.0, 9, 1))
    for x, y in zip(g1, g2):
        assert np.array_equal(x, y)


def test_p14_dropout_gradients_match_finite_differences():
    """With the keep decisions fixed (they depend on positions, seed and offset only), the
    dropout backward is the exact gradient of the dropout forward: central differences in
    fp64 for q, k, v and the sink."""
    p = W.random_problem(141, [6, 4], [7, 4], 4, 2, 4, 3, True, window_left=4, dtype="fp32", with_dout=True)
    drop = (0.3, 77, 5)
    a = (p.cu_seqlens_q, p.cu_seqlens_k)
    loss = lambda q, k, v, s: float((ref.fwd(q, k, v, *a, s, p.softmax_scale, True, 4, -1, drop)[0] * p.dout).sum())
    dq, dk, dv, ds = ref.bwd(p.q, p.k, p.v, p.dout, *a, p.sink, p.softmax_scale, True, 4, -1, drop)
    base = [p.q.astype(np.float64), p.k.astype(np.float64), p.v.astype(np.float64), p.sink.astype(np.float64)]
    h = 1e-6
    for which, grad in enumerate((dq, dk, dv, ds)):
        x = base[which]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if i == which else base[i] for i in range(4)]
            args_m = [xm if i == which else base[i] for i in range(4)]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.abs(num - grad).max() / max(1e-12, np.abs(grad).max())
        assert err < 1e-6, (which, err)


def test_p14_dropout_is_unbiased_on_average():
    """Averaged over seeds, the dropout output approaches the output without dropout."""
    p = W.random_problem(142, [8], [8], 2, 2, 4, 4, True, dtype="fp32")
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True)
    o_ref, _ = ref.fwd(p.q, p.k, p.v, *a)
    n = 400
    outs = np.stack([ref.fwd(p.q, p.k, p.v, *a, dropout=(0.5, 1000 + s, 0))[0] for s in range(n)])
    se = outs.std(axis=0) / math.sqrt(n)          # standard error of each element's mean
    assert np.all(np.abs(outs.mean(axis=0) - o_ref) <= 5 * se + 1e-12)
