"""Sink-attention oracle: a plain, slow, float64 CPU implementation.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import this module.  The
CUDA path never imports it, shares no code with it, and has no CPU fallback.

Every function materialises the full score matrix of one (sequence, head) and writes
the definition out with NumPy float64 arrays; no blocking, fusion or online rescaling.
Sources, by page and section:

* Sink softmax -- Huawei CANN ops-transformer ``flash_attn`` operator doc, section
  "Function", the formula after "After adding sink": S = QK^T * scale,
  m = max(sink, max S), out = sum_j e^{S_j - m} v_j / (sum_j e^{S_j - m} + e^{sink - m}).
* Returned LSE -- same doc, the ``softmax_lse`` formula (log of the sum of e^{S - max S},
  plus max S: the sink is NOT included) and the ``softmax_lse`` note ("float32",
  shape (Q_N, Q_T) for the TND layout).
* Learnable offset -- slime ``learnable_softmax_attention.py``, module docstring: the
  offset is an extra logit column appended to the scaled scores, equivalently
  softmax(S) * sigmoid(lse - offset).  The offset is the sink, in post-scale units.
* softmax_n -- Flash-Attention-Softmax-N README, first section: exp(x_i)/(n + sum exp x_j),
  i.e. sink = log n.
* Bottom-right causal alignment -- PyTorch issue #108108, "Proposal" and "Benefits":
  query row i of sq sees key j iff j <= i + (sk - sq); an all-masked row outputs zero.
* Sliding window (left, right), -1 = unbounded -- slime wrapper docstring ("window_size");
  CANN doc, "Mask Parameter Group" (win_left / win_right, -1 = positive infinity).
* GQA -- CANN doc, "Common Parameter Group" (Q_N % KV_N == 0); q head h reads kv head
  h // (Q_N / KV_N).
* Packed THD varlen with cu_seqlens -- slime wrapper docstring; CANN doc,
  "SeqLengths Parameter Group".
* Backward -- the exact gradient of the forward above.  slime's class docstring and
  ``backward`` state the same result in another form (dS = P_van * s * (dP - s * di),
  d_offset = -sum (dO . O_van) s (1 - s)); the tests check that form against this one.
* Decode split + LSE merge -- CANN doc, the ``softmax_lse`` note (partial results of
  ring attention are combined through max / sum / log); the sink enters once, after
  the partials are combined.
* Dropout -- slime wrapper (``dropout_p`` passed to flash attention, whose probabilities
  are then scaled by sigmoid(lse - offset)): dropout applies to the sink-normalised
  probabilities, kept ones scaled so the expectation is unchanged, lse untouched.  The keep
  decisions come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
  As Easy as 1, 2, 3", SC 2011), on the counter layout ``dropout_keep`` defines.
* Paged K/V -- CANN doc, "Paged Attention Parameter Group" (block_table (B,
  max_num_blocks_per_seq) int32, block_size in [16, 1024] and a multiple of 16, seqused_kv)
  and the PA_BBND layout of k / v, (num_blocks, block_size, KV_N, D).

Readings where the pages are silent: a row with no visible
key has lse = -inf; with sink = -inf as well its output is 0; the window is measured
from the bottom-right diagonal and causal clamps right to min(right, 0).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def allowed_mask(sq: int, sk: int, causal: bool, window_left: int = -1,
                 window_right: int = -1) -> np.ndarray:
    """Visible (query, key) pairs of one sequence, bottom-right aligned.  bool [sq, sk].

    Query row i sits at key position i + (sk - sq) (PyTorch issue #108108, Proposal).
    It sees key j when  i + off - left <= j <= i + off + right, with an unbounded side
    for -1, and causal meaning right = min(right, 0).
    """
    off = sk - sq
    right = np.inf if window_right < 0 else float(window_right)
    if causal:
        right = min(right, 0.0)
    left = np.inf if window_left < 0 else float(window_left)
    i = np.arange(sq, dtype=np.float64)[:, None]
    j = np.arange(sk, dtype=np.float64)[None, :]
    return (j <= i + off + right) & (j >= i + off - left)


def attend_head(qh, kh, vh, sink_h: float, scale: float, allowed: np.ndarray,
                drop: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Forward of one (sequence, head): the CANN sink formula, written out.

    qh [sq, dk], kh [sk, dk], vh [sk, dv]; sink_h a float (may be -inf).  drop, when given,
    is the dropout weight Z [sq, sk] (keep mask x 256 / T): out = (P o Z) V.
    Returns out [sq, dv], lse [sq] (vanilla: sink excluded), P [sq, sk],
    p_sink [sq] (the probability the sink column takes), S [sq, sk].
    """
    qh, kh, vh = _f64(qh), _f64(kh), _f64(vh)
    sq, sk = allowed.shape
    sink_h = float(sink_h)
    S = float(scale) * (qh @ kh.T)                                   # S = Q K^T * scale
    S_vis = np.where(allowed, S, NEG_INF)
    smax = S_vis.max(axis=1) if sk > 0 else np.full(sq, NEG_INF)      # max S over visible keys
    m = np.maximum(smax, sink_h)                                      # m = max(sink, max S)
    m_ref = np.where(np.isfinite(m), m, 0.0)    # m = -inf only when nothing is visible at all
    with np.errstate(invalid="ignore", over="ignore"):
        E = np.exp(S_vis - m_ref[:, None])                            # e^{S - m}, 0 where masked
        e_sink = np.exp(sink_h - m_ref)                               # e^{sink - m}
    den = E.sum(axis=1) + e_sink
    inv = np.where(den > 0, 1.0 / np.where(den > 0, den, 1.0), 0.0)
    P = E * inv[:, None]
    p_sink = e_sink * inv
    out = (P if drop is None else P * drop) @ vh
    # vanilla lse: log sum_j e^{S_j - max S} + max S over the visible keys
    with np.errstate(divide="ignore", invalid="ignore"):
        smax_ref = np.where(np.isfinite(smax), smax, 0.0)
        z = np.exp(S_vis - smax_ref[:, None]).sum(axis=1)
        lse = np.where(np.isfinite(smax), np.log(z) + smax_ref, NEG_INF)
    return {"out": out, "lse": lse, "P": P, "p_sink": p_sink, "S": S}


# --- dropout --------------------------------------------------------------------------

PHILOX_M = (0xD2511F53, 0xCD9E8D57)   # round multipliers of Philox4x32 (Salmon et al. 2011)
PHILOX_W = (0x9E3779B9, 0xBB67AE85)   # key increments (Weyl sequence) of Philox4x32
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds on numpy arrays of 32-bit values (held as uint64).
    ctr: 4 arrays (or ints), key: 2 arrays (or ints); returns the 4 output words."""
    c = [np.asarray(x, dtype=np.uint64) & _U32 for x in ctr]
    k = [np.asarray(x, dtype=np.uint64) & _U32 for x in key]
    for _ in range(10):
        p0 = np.uint64(PHILOX_M[0]) * c[0]
        p1 = np.uint64(PHILOX_M[1]) * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _U32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _U32
        c = [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]
        k = [(k[0] + np.uint64(PHILOX_W[0])) & _U32, (k[1] + np.uint64(PHILOX_W[1])) & _U32]
    return c


def dropout_threshold(p: float) -> int:
    """Keep threshold T: an element is kept when its random byte is below T, so the keep
    probability is T / 256.  T = floor(256 (1 - p) + 1/2) for the float32 value of p (the
    call passes p as a float), evaluated exactly (halves round up); 1 <= T <= 256."""
    t = int(math.floor(256.0 * (1.0 - float(np.float32(p))) + 0.5))
    if not 1 <= t <= 256:
        raise ValueError("dropout p must satisfy 1 <= round(256 (1 - p)) <= 256")
    return t


def dropout_keep(seed: int, offset: int, threshold: int, rows, head: int, nkeys: int) -> np.ndarray:
    """Keep mask [len(rows), nkeys] of query rows `rows` (packed row indices) of q head
    `head` against keys 0 .. nkeys-1 of their sequence.  Key j of row r uses byte j % 16 of
    Philox4x32-10 with counter (j // 16, r, head, offset) and key (seed low 32 bits, seed
    high 32 bits); byte t is bits 8 (t % 4) .. 8 (t % 4) + 7 of output word t // 4."""
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    j = np.arange(nkeys, dtype=np.uint64)[None, :]
    words = philox4x32_10((j >> np.uint64(4), rows, head, offset), (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    t = j & np.uint64(15)
    w = np.choose((t >> np.uint64(2)).astype(np.int64), [np.broadcast_to(x, np.broadcast(rows, j).shape) for x in words])
    byte = (w >> (np.uint64(8) * (t & np.uint64(3)))) & np.uint64(0xFF)
    return byte < np.uint64(threshold)


def _sink_of(sink: Optional[np.ndarray], h: int) -> float:
    return NEG_INF if sink is None else float(sink[h])


def _seq_ranges(cu: np.ndarray, b: int) -> Tuple[int, int]:
    return int(cu[b]), int(cu[b + 1])


def _drop_weights(dropout, q0: int, q1: int, h: int, nkeys: int) -> Optional[np.ndarray]:
    """Dropout weights Z [q1 - q0, nkeys] (keep x 256 / T) of rows q0 .. q1-1 of head h, or
    None without dropout.  dropout = (p, seed, offset)."""
    if dropout is None:
        return None
    p, seed, offset = dropout
    t = dropout_threshold(p)
    keep = dropout_keep(seed, offset, t, np.arange(q0, q1), h, nkeys)
    return keep * (256.0 / t)


def fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, sink, softmax_scale: float, causal: bool = False,
        window_left: int = -1, window_right: int = -1, dropout=None) -> Tuple[np.ndarray, np.ndarray]:
    """Packed THD forward.  q [T_q,Hq,dk], k [T_k,Hkv,dk], v [T_k,Hkv,dv], sink [Hq] or None.
    dropout = (p, seed, offset) or None.

    Returns out [T_q, Hq, dv] float64 and lse [Hq, T_q] float64 (vanilla lse).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    tq, hq, _ = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    group = hq // hkv
    out = np.zeros((tq, hq, dv))
    lse = np.full((hq, tq), NEG_INF)
    for b in range(len(cu_seqlens_q) - 1):
        q0, q1 = _seq_ranges(cu_seqlens_q, b)
        k0, k1 = _seq_ranges(cu_seqlens_k, b)
        if q1 == q0:
            continue
        mask = allowed_mask(q1 - q0, k1 - k0, causal, window_left, window_right)
        for h in range(hq):
            r = attend_head(q[q0:q1, h], k[k0:k1, h // group], v[k0:k1, h // group],
                            _sink_of(sink, h), softmax_scale, mask,
                            _drop_weights(dropout, q0, q1, h, k1 - k0))
            out[q0:q1, h] = r["out"]
            lse[h, q0:q1] = r["lse"]
    return out, lse


def bwd_head(qh, kh, vh, dout_h, sink_h: float, scale: float, allowed: np.ndarray,
             drop: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Gradients of one (sequence, head) for the loss sum(dout * out).

    With P the sink-normalised probabilities and p_sink the sink's share of each row:
      dP = dO V^T,  D_i = dO_i . out_i,  dS = P * (dP - D),
      dq = scale dS K,  dk = scale dS^T Q,  dv = P^T dO,  d_sink = -sum_i p_sink_i D_i.
    With dropout weights Z (out = (P o Z) V): dP = Z o (dO V^T) and dv = (P o Z)^T dO; D and
    the rest are unchanged (D = dO . out still equals sum_j P_ij dP_ij).
    """
    r = attend_head(qh, kh, vh, sink_h, scale, allowed, drop)
    qh, kh, vh, do = _f64(qh), _f64(kh), _f64(vh), _f64(dout_h)
    P, out = r["P"], r["out"]
    PZ = P if drop is None else P * drop
    dP = do @ vh.T
    if drop is not None:
        dP = dP * drop
    D = (do * out).sum(axis=1)
    dS = P * (dP - D[:, None])
    return {
        "dq": float(scale) * (dS @ kh),
        "dk": float(scale) * (dS.T @ qh),
        "dv": PZ.T @ do,
        "dsink": -float((r["p_sink"] * D).sum()),
        "D": D, "out": out, "lse": r["lse"],
    }


def bwd(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, sink, softmax_scale: float,
        causal: bool = False, window_left: int = -1, window_right: int = -1, dropout=None):
    """Packed THD backward.  Returns dq, dk, dv (float64, input layouts) and dsink [Hq].
    dropout = (p, seed, offset) or None (the forward's keep decisions are drawn again).

    dk / dv of a kv head sum the contributions of the q heads of its group.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    hq, hkv = q.shape[1], k.shape[1]
    group = hq // hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dsink = np.zeros(hq)
    for b in range(len(cu_seqlens_q) - 1):
        q0, q1 = _seq_ranges(cu_seqlens_q, b)
        k0, k1 = _seq_ranges(cu_seqlens_k, b)
        if q1 == q0:
            continue
        mask = allowed_mask(q1 - q0, k1 - k0, causal, window_left, window_right)
        for h in range(hq):
            g = h // group
            r = bwd_head(q[q0:q1, h], k[k0:k1, g], v[k0:k1, g], dout[q0:q1, h],
                         _sink_of(sink, h), softmax_scale, mask,
                         _drop_weights(dropout, q0, q1, h, k1 - k0))
            dq[q0:q1, h] = r["dq"]
            dk[k0:k1, g] += r["dk"]
            dv[k0:k1, g] += r["dv"]
            dsink[h] += r["dsink"]
    return dq, dk, dv, dsink


def decode(q, k, v, cu_seqlens_k, sink, softmax_scale: float, causal: bool = True,
           window_left: int = -1, window_right: int = -1):
    """Decode: q [B, Hq, dk], one query per sequence.  Returns out [B, Hq, dv], lse [Hq, B]."""
    q = _f64(q)
    b = q.shape[0]
    cu_q = np.arange(b + 1, dtype=np.int64)
    return fwd(q, k, v, cu_q, cu_seqlens_k, sink, softmax_scale, causal, window_left, window_right)


def gather_paged(cache, block_table, seqused_k, block_size: int):
    """Keys (or values) of each sequence read through its block-table row: key t of
    sequence b is row t % block_size of block block_table[b, t // block_size] of a cache
    [num_blocks, block_size, H, d] (CANN flash_attn doc, "Paged Attention Parameter Group";
    the PA_BBND layout (num_blocks, block_size, KV_N, D) of its parameter table).
    Returns the packed rows [sum seqused_k, H, d] and their cu_seqlens."""
    cache = np.asarray(cache)
    table = np.asarray(block_table)
    used = [int(n) for n in np.asarray(seqused_k)]
    rows = []
    for b, n in enumerate(used):
        t = np.arange(n)
        rows.append(cache[table[b, t // block_size], t % block_size])
    cu = np.zeros(len(used) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(used)
    packed = np.concatenate(rows, axis=0) if rows else cache[:0, 0]
    return packed, cu


def decode_paged(q, k_cache, v_cache, block_table, seqused_k, block_size: int, sink,
                 softmax_scale: float, causal: bool = True, window_left: int = -1,
                 window_right: int = -1):
    """Decode over a paged K/V cache: the plain decode of the keys and values each
    sequence's block-table row names.  Returns out [B, Hq, dv], lse [Hq, B]."""
    k, cu = gather_paged(k_cache, block_table, seqused_k, block_size)
    v, _ = gather_paged(v_cache, block_table, seqused_k, block_size)
    return decode(q, k, v, cu, sink, softmax_scale, causal, window_left, window_right)


# --- split-KV partials and the LSE merge --------------------------------------------

def split_bounds(sk: int, num_splits: int) -> List[Tuple[int, int]]:
    """Contiguous key chunks [lo, hi) covering [0, sk), num_splits of them (last may be short)."""
    num_splits = max(1, int(num_splits))
    size = -(-sk // num_splits) if sk > 0 else 0
    return [(min(c * size, sk), min((c + 1) * size, sk)) for c in range(num_splits)]


def decode_partials(q_row, kh, vh, scale: float, allowed_row: np.ndarray, num_splits: int):
    """Per key chunk: local max m_c, local sum l_c = sum e^{S - m_c}, unnormalised
    o_c = sum e^{S - m_c} v (no sink in any chunk).  A chunk with no visible key has
    m_c = -inf, l_c = 0, o_c = 0."""
    q_row, kh, vh = _f64(q_row), _f64(kh), _f64(vh)
    S = float(scale) * (kh @ q_row)
    parts = []
    for lo, hi in split_bounds(kh.shape[0], num_splits):
        vis = allowed_row[lo:hi]
        if hi <= lo or not vis.any():
            parts.append((NEG_INF, 0.0, np.zeros(vh.shape[1])))
            continue
        s = S[lo:hi][vis]
        m_c = s.max()
        e = np.exp(s - m_c)
        parts.append((m_c, e.sum(), e @ vh[lo:hi][vis]))
    return parts


def merge_partials(parts, sink_h: float) -> Tuple[np.ndarray, float]:
    """Combine chunk partials, then apply the sink once.

    m = max(sink, max_c m_c);  den = sum_c l_c e^{m_c - m} + e^{sink - m};
    out = sum_c o_c e^{m_c - m} / den;  lse = log sum_c l_c e^{m_c - M} + M, M = max_c m_c.
    """
    ms = np.array([p[0] for p in parts], dtype=np.float64)
    ls = np.array([p[1] for p in parts], dtype=np.float64)
    os_ = np.stack([p[2] for p in parts])
    M = ms.max()
    m = max(M, float(sink_h))
    if not np.isfinite(m):
        return np.zeros(os_.shape[1]), NEG_INF
    w = np.where(np.isfinite(ms), np.exp(np.where(np.isfinite(ms), ms, 0.0) - m), 0.0)
    den = (ls * w).sum() + np.exp(float(sink_h) - m)
    out = (os_ * w[:, None]).sum(axis=0) / den
    if np.isfinite(M):
        wM = np.where(np.isfinite(ms), np.exp(np.where(np.isfinite(ms), ms, 0.0) - M), 0.0)
        lse = float(np.log((ls * wM).sum()) + M)
    else:
        lse = NEG_INF
    return out, lse


# --- sampled checks at full size ------------------------------------------------------

def fwd_rows(q, k, v, cu_seqlens_q, cu_seqlens_k, sink, softmax_scale: float, causal: bool,
             window_left: int, window_right: int, b: int, h: int, rows: Sequence[int], dropout=None):
    """out [len(rows), dv] and lse [len(rows)] for chosen query rows (sequence-local
    indices) of sequence b, q head h; identical arithmetic to ``fwd`` (dropout included:
    the keep decisions of exactly those packed rows)."""
    q0, q1 = _seq_ranges(cu_seqlens_q, b)
    k0, k1 = _seq_ranges(cu_seqlens_k, b)
    hq, hkv = q.shape[1], k.shape[1]
    g = h // (hq // hkv)
    rows = np.asarray(rows, dtype=np.int64)
    full = allowed_mask(q1 - q0, k1 - k0, causal, window_left, window_right)
    drop = None
    if dropout is not None:
        p, seed, offset = dropout
        t = dropout_threshold(p)
        drop = dropout_keep(seed, offset, t, q0 + rows, h, k1 - k0) * (256.0 / t)
    r = attend_head(_f64(q[q0 + rows, h]), _f64(k[k0:k1, g]), _f64(v[k0:k1, g]),
                    _sink_of(sink, h), softmax_scale, full[rows], drop)
    return r["out"], r["lse"]


def bwd_sequence_group(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, sink, softmax_scale: float,
                       causal: bool, window_left: int, window_right: int, b: int, g: int, dropout=None):
    """Backward restricted to sequence b and kv head g (all q heads of its group).

    Returns dq [sq, G, dk] for those q heads, dk [sk, dk] and dv [sk, dv] of kv head g,
    and dsink contributions [G] of sequence b -- identical arithmetic to ``bwd``."""
    q0, q1 = _seq_ranges(cu_seqlens_q, b)
    k0, k1 = _seq_ranges(cu_seqlens_k, b)
    hq, hkv = q.shape[1], k.shape[1]
    group = hq // hkv
    mask = allowed_mask(q1 - q0, k1 - k0, causal, window_left, window_right)
    dq = np.zeros((q1 - q0, group, q.shape[2]))
    dk = np.zeros((k1 - k0, k.shape[2]))
    dv = np.zeros((k1 - k0, v.shape[2]))
    ds = np.zeros(group)
    for hh in range(group):
        h = g * group + hh
        r = bwd_head(q[q0:q1, h], k[k0:k1, g], v[k0:k1, g], dout[q0:q1, h], _sink_of(sink, h),
                     softmax_scale, mask, _drop_weights(dropout, q0, q1, h, k1 - k0))
        dq[:, hh] = r["dq"]
        dk += r["dk"]
        dv += r["dv"]
        ds[hh] = r["dsink"]
    return dq, dk, dv, ds


def pair_count(cu_seqlens_q, cu_seqlens_k, num_heads_q: int, causal: bool, window_left: int = -1,
               window_right: int = -1) -> int:
    """Number of visible (query, key, q head) triples: the unit the flop counts use."""
    total = 0
    for b in range(len(cu_seqlens_q) - 1):
        sq = int(cu_seqlens_q[b + 1] - cu_seqlens_q[b])
        sk = int(cu_seqlens_k[b + 1] - cu_seqlens_k[b])
        if sq and sk:
            total += int(allowed_mask(sq, sk, causal, window_left, window_right).sum())
    return total * int(num_heads_q)
