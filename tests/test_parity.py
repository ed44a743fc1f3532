"""Parity of the CUDA path with the fp64 oracle on small seeded problems: every output
element compared, shapes spanning several 128-row tiles with ragged tails, plus the
degenerate cases (empty sequences, rows that see no key, sq > sk, sink = -inf)."""
import math
import zlib

import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_grad, check_lse, check_out, to_np

pytestmark = pytest.mark.gpu

try:
    from gpu_util import run_bwd, run_decode, run_fwd
except Exception:  # torch without CUDA still imports; the calls fail at run time
    pass


def _seed(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


def _oracle_fwd(p):
    return ref.fwd(p.q, p.k, p.v, p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale,
                   p.causal, p.window_left, p.window_right)


_LENS_A = [int(n) for n in np.random.default_rng(11).integers(0, 700, size=40)] + [0, 1]
_LENS_B = [int(n) for n in np.random.default_rng(12).integers(1, 900, size=30)]
_LENS_C = [int(n) for n in np.random.default_rng(13).integers(0, 5, size=9000)]
# 600 short sequences: the item table leaves no room for the forward's output staging area,
# so the persistent forward stores rows directly from registers.
_LENS_D = [int(n) for n in np.random.default_rng(43).integers(0, 300, size=600)]

FWD_CASES = [
    # name, lens_q, lens_k, hq, hkv, dk, dv, causal, wl, wr, sink, dtype
    ("full_d128", [300, 300], [300, 300], 4, 4, 128, 128, False, -1, -1, "normal", "bf16"),
    ("causal_d128", [300, 300], [300, 300], 4, 4, 128, 128, True, -1, -1, "normal", "bf16"),
    ("varlen_gqa_causal", [1, 127, 128, 129, 0, 333, 500], [1, 127, 128, 129, 0, 333, 500],
     8, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    ("sq_ne_sk_causal", [5, 100, 200, 7], [2, 300, 150, 0], 4, 2, 128, 128, True, -1, -1,
     "normal", "bf16"),
    ("window_causal", [400, 257], [400, 300], 4, 1, 128, 128, True, 64, 0, "normal", "bf16"),
    ("window_two_sided", [300], [350], 2, 2, 128, 128, False, 32, 16, "uniform", "bf16"),
    ("dk64_dv32_window", [300, 129], [333, 200], 2, 1, 64, 32, True, 100, 0, "normal", "bf16"),
    ("dk64_dv64", [257, 64], [257, 64], 4, 2, 64, 64, False, -1, -1, "normal", "bf16"),
    ("dk128_dv64", [200, 3], [260, 300], 4, 4, 128, 64, True, -1, -1, "normal", "bf16"),
    ("dk64_dv128", [130], [130], 2, 2, 64, 128, True, -1, -1, "normal", "bf16"),
    ("dk128_dv32", [190], [190], 2, 1, 128, 32, False, -1, -1, "normal", "bf16"),
    ("no_sink", [300, 40], [300, 40], 4, 2, 128, 128, True, -1, -1, None, "bf16"),
    ("neg_inf_sink", [5, 260], [2, 260], 4, 2, 128, 128, True, -1, -1, "neg_inf", "bf16"),
    ("big_sink", [150], [150], 2, 2, 128, 128, True, -1, -1, [8.0, -8.0], "bf16"),
    ("fp32_causal_gqa", [70, 1, 130], [90, 5, 130], 4, 2, 128, 64, True, -1, -1, "normal", "fp32"),
    ("fp32_window", [100], [120], 2, 2, 64, 32, True, 20, 0, "normal", "fp32"),
    ("fp32_full_d64", [65, 33], [65, 200], 2, 1, 64, 64, False, -1, -1, "uniform", "fp32"),
    # More work items than SMs, so the persistent forward's CTAs each take several items of
    # mixed cost (zero-length and one-row sequences included): row-tile pairs of one head
    # (odd group), head pairs (even group), and keys longer than queries with a window.
    ("persistent_odd_group", _LENS_A, _LENS_A, 6, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    ("persistent_even_group", _LENS_B, _LENS_B, 8, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    ("persistent_window_sk_gt_sq", _LENS_A, [n + 37 for n in _LENS_A], 4, 4, 128, 64, True, 200, 0,
     "uniform", "bf16"),
    # fp16 inputs on the tensor-core path (both unit arrangements) and on the CUDA-core one
    ("fp16_causal_gqa", _LENS_B[:8], _LENS_B[:8], 8, 2, 128, 128, True, -1, -1, "normal", "fp16"),
    ("fp16_odd_group_window", [300, 129], [333, 200], 3, 1, 128, 64, True, 100, 0, "normal", "fp16"),
    ("fp16_dk64", [257, 64], [257, 64], 4, 2, 64, 64, False, -1, -1, "uniform", "fp16"),
    # dv = 32 on the tensor cores: 64-wide PV over zero-filled V columns, 32 columns stored
    ("fp16_dv32", [190], [190], 2, 1, 128, 32, True, -1, -1, "normal", "fp16"),
    ("dk64_dv32_varlen_gqa", [1, 127, 0, 129, 333], [1, 127, 0, 129, 340], 8, 2, 64, 32, True, -1, -1,
     "normal", "bf16"),
    ("dk64_dv32_odd_group_persistent", _LENS_A, _LENS_A, 3, 1, 64, 32, True, 200, 0, "uniform", "bf16"),
    ("dk128_dv32_sq_ne_sk", [5, 100, 200, 7], [2, 300, 150, 0], 4, 2, 128, 32, True, -1, -1, "normal", "bf16"),
    # 9000 sequences: the item table would not fit in shared memory, so the forward runs one
    # CTA per item of the dense grid instead.
    ("grid_mode_many_sequences", _LENS_C, _LENS_C, 2, 1, 128, 128, True, -1, -1, "normal", "bf16"),
    ("persistent_unstaged", _LENS_D, _LENS_D, 4, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    # head dim 256: the one-unit tensor-core forward (Q in TMEM, 64-key tiles), its fp16
    # variant, and the CUDA-core kernel for fp32
    ("d256_causal_gqa", [1, 63, 64, 65, 0, 300, 700], [1, 63, 64, 65, 0, 300, 700], 8, 2, 256, 256,
     True, -1, -1, "normal", "bf16"),
    ("d256_sq_ne_sk_full", [5, 200, 129], [2, 333, 150], 4, 4, 256, 256, False, -1, -1, "uniform", "bf16"),
    ("d256_window_neg_inf_sink", [400, 3], [420, 260], 4, 1, 256, 256, True, 100, 0, "neg_inf", "bf16"),
    ("d256_fp16_causal", [300, 257], [300, 257], 4, 2, 256, 256, True, -1, -1, "normal", "fp16"),
    ("d256_fp32", [70, 33], [90, 33], 2, 1, 256, 256, True, -1, -1, "normal", "fp32"),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fwd_matches_oracle(case):
    name, lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype = case
    p = W.random_problem(_seed(name), lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype)
    out, lse = run_fwd(p)
    ro, rl = _oracle_fwd(p)
    check_out(to_np(out), ro, dtype)
    check_lse(to_np(lse), rl, dtype)


def test_fwd_is_deterministic():
    """Two runs of the same forward give the same bits (no atomics, fixed item order)."""
    p = W.random_problem(7, _LENS_B, _LENS_B, 8, 2, 128, 128, True)
    o1, l1 = run_fwd(p)
    o2, l2 = run_fwd(p)
    assert np.array_equal(to_np(o1), to_np(o2)) and np.array_equal(to_np(l1), to_np(l2))


def test_fwd_softmax_n_and_vanilla_identity():
    """sink = log n equals softmax_n; the GPU result for n -> sink = log n agrees with oracle."""
    for n in (1.0, 0.5, 3.0):
        p = W.random_problem(21, [200], [230], 1, 1, 64, 32, True, 50, 0, math.log(n))
        out, lse = run_fwd(p)
        ro, rl = _oracle_fwd(p)
        check_out(to_np(out), ro, "bf16")
        check_lse(to_np(lse), rl, "bf16")


def test_fwd_fully_masked_rows_are_zero():
    # q=5, k=2 causal: rows 0-2 see nothing -> out exactly 0, lse = -inf
    p = W.random_problem(22, [5, 4], [2, 0], 2, 1, 128, 128, True)
    out, lse = run_fwd(p)
    o, l = to_np(out), to_np(lse)
    dead = [0, 1, 2, 5, 6, 7, 8]
    assert np.all(o[dead] == 0.0)
    assert np.all(np.isneginf(l[:, dead]))


BWD_CASES = [
    ("causal_d128", [300, 200], [300, 200], 4, 4, 128, 128, True, -1, -1, "normal", "bf16"),
    ("varlen_gqa", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    ("sq_ne_sk", [5, 130], [2, 200], 4, 2, 128, 128, True, -1, -1, "normal", "bf16"),
    ("window", [260], [300], 2, 1, 128, 128, True, 50, 0, "normal", "bf16"),
    ("full_noncausal", [200], [170], 2, 2, 128, 128, False, -1, -1, "uniform", "bf16"),
    ("dk64_dv32", [150, 90], [160, 90], 2, 1, 64, 32, True, 40, 0, "normal", "bf16"),
    ("no_sink", [190], [190], 2, 2, 128, 64, True, -1, -1, None, "bf16"),
    ("dk64_dv64_gqa", [300, 131], [300, 131], 4, 1, 64, 64, True, -1, -1, "normal", "bf16"),
    ("dk64_dv128", [257], [300], 2, 2, 64, 128, True, -1, -1, "uniform", "bf16"),
    ("gqa4_long_window", [700, 300], [700, 300], 8, 2, 128, 128, True, 200, 0, "normal", "bf16"),
    ("neg_inf_sink_masked_rows", [5, 260], [2, 260], 4, 2, 128, 128, True, -1, -1, "neg_inf", "bf16"),
    ("fp32_gqa", [70, 33], [80, 33], 4, 2, 128, 64, True, -1, -1, "normal", "fp32"),
    ("fp32_window", [90], [90], 2, 2, 64, 64, False, 10, 5, "normal", "fp32"),
    ("fp16_varlen_gqa", [1, 129, 0, 257], [1, 129, 0, 257], 8, 2, 128, 128, True, -1, -1, "normal", "fp16"),
    ("fp16_dv64_window", [260], [300], 2, 1, 128, 64, True, 50, 0, "normal", "fp16"),
    ("fp16_dk64", [300, 131], [300, 131], 4, 1, 64, 64, True, -1, -1, "normal", "fp16"),
    ("fp16_dv32", [150, 90], [160, 90], 2, 1, 64, 32, True, 40, 0, "normal", "fp16"),
    ("dk64_dv32_varlen_gqa", [1, 129, 0, 257], [1, 129, 0, 300], 8, 2, 64, 32, True, -1, -1, "normal", "bf16"),
    ("dk128_dv32_gqa_window", [300, 131], [333, 131], 4, 1, 128, 32, True, 100, 0, "normal", "bf16"),
    ("dk128_dv32_full", [200, 65], [170, 65], 2, 2, 128, 32, False, -1, -1, "uniform", "fp16"),
    # head dim 256: the dQ / dK / dV tensor-core kernels (bf16, fp16); fp32 on the CUDA cores
    ("d256_causal_gqa", [1, 100, 0, 131], [1, 100, 0, 131], 4, 2, 256, 256, True, -1, -1, "normal", "bf16"),
    ("d256_fp16_window", [120], [150], 2, 2, 256, 256, True, 40, 0, "normal", "fp16"),
    ("d256_sq_ne_sk_full", [5, 130], [2, 200], 4, 2, 256, 256, False, -1, -1, "uniform", "bf16"),
    ("d256_long_gqa4_window", [700, 300], [700, 300], 8, 2, 256, 256, True, 200, 0, "normal", "bf16"),
    ("d256_neg_inf_sink_masked_rows", [5, 260], [2, 260], 4, 2, 256, 256, True, -1, -1, "neg_inf", "bf16"),
    ("d256_fp32", [40, 9], [50, 9], 2, 1, 256, 256, True, -1, -1, "normal", "fp32"),
]


@pytest.mark.parametrize("deterministic", [False, True], ids=["atomic_dq", "deterministic"])
@pytest.mark.parametrize("case", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_matches_oracle(case, deterministic):
    name, lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype = case
    p = W.random_problem(_seed(name) + 7, lq, lk, hq, hkv, dk, dv, causal, wl, wr, sink,
                         dtype, with_dout=True)
    out, lse, dq, dk_, dv_, ds = run_bwd(p, deterministic)
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, p.causal, wl, wr)
    rdq, rdk, rdv, rds = ref.bwd(p.q, p.k, p.v, p.dout, *a)
    check_grad(to_np(dq), rdq, dtype, "dq")
    check_grad(to_np(dk_), rdk, dtype, "dk")
    check_grad(to_np(dv_), rdv, dtype, "dv")
    if p.sink is not None:
        check_grad(to_np(ds), rds, dtype, "dsink")


def test_bwd_fully_masked_rows_have_zero_dq():
    p = W.random_problem(23, [5, 3], [2, 0], 2, 1, 128, 128, True, with_dout=True)
    out, lse, dq, dk, dv, ds = run_bwd(p)
    assert np.all(to_np(dq)[[0, 1, 2, 5, 6, 7]] == 0.0)
    assert np.all(np.isfinite(to_np(ds)))


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "bf16_d256"])
def test_bwd_deterministic_is_bitwise_repeatable(dtype):
    """The deterministic backward gives the same bits on every run (dq summed over 7 key
    tiles in a fixed order, GQA heads, a sink); its results match the atomic path within
    the gradient tolerance."""
    d = 256 if dtype.endswith("d256") else 128
    dtype = dtype.split("_")[0]
    p = W.random_problem(31, [900, 300], [900, 300], 8, 2, d, d, True, dtype=dtype, with_dout=True)
    runs = [run_bwd(p, True) for _ in range(3)]
    for name, idx in (("dq", 2), ("dk", 3), ("dv", 4), ("dsink", 5)):
        first = to_np(runs[0][idx])
        for r in runs[1:]:
            assert np.array_equal(first, to_np(r[idx])), f"{name} differs between runs"
    fast = run_bwd(p, False)
    check_grad(to_np(runs[0][2]), to_np(fast[2]), dtype, "dq vs atomic dq")



DECODE_CASES = [
    # name, lens_k, hq, hkv, dk, dv, causal, wl, wr, sink, splits
    ("gqa8_auto", [1, 63, 64, 65, 1000, 4097], 16, 2, 128, 128, True, -1, -1, "normal", 0),
    ("gqa8_splits1", [700, 33], 16, 2, 128, 128, True, -1, -1, "normal", 1),
    ("gqa8_splits7", [700, 1, 2049], 8, 1, 128, 128, True, -1, -1, "uniform", 7),
    ("mha", [300, 129], 4, 4, 128, 128, True, -1, -1, "normal", 3),
    ("gqa24_two_head_blocks", [500, 17], 24, 1, 128, 128, True, -1, -1, "normal", 0),
    ("window_left", [900, 50], 8, 2, 128, 128, True, 100, 0, "normal", 4),
    ("dk64_dv32", [333, 1000], 8, 2, 64, 32, True, -1, -1, "normal", 0),
    ("dk128_dv64", [333], 8, 1, 128, 64, True, -1, -1, "normal", 2),
    ("no_sink", [257, 65], 8, 2, 128, 128, True, -1, -1, None, 0),
    ("neg_inf_sink_empty_seq", [0, 70], 8, 2, 128, 128, True, -1, -1, "neg_inf", 0),
    ("fp32", [300, 41], 8, 2, 128, 64, True, -1, -1, "normal", 0),
    ("fp16_gqa8", [1, 63, 1000, 4097], 16, 2, 128, 128, True, -1, -1, "normal", 0),
    ("fp16_dk64_dv32", [333, 1000], 8, 2, 64, 32, True, -1, -1, "normal", 3),
    ("d256_gqa8", [1, 63, 700, 3000], 16, 2, 256, 256, True, -1, -1, "normal", 0),
    ("fp16_d256_splits3", [500, 65], 8, 1, 256, 256, True, -1, -1, "normal", 3),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_matches_oracle(case):
    name, lk, hq, hkv, dk, dv, causal, wl, wr, sink, splits = case
    dtype = name.split("_")[0] if name.split("_")[0] in ("fp32", "fp16") else "bf16"
    d = W.random_decode(_seed(name) + 3, lk, hq, hkv, dk, dv, causal, wl, wr, sink, dtype)
    out, lse = run_decode(d, splits)
    ro, rl = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale, causal, wl, wr)
    check_out(to_np(out), ro, dtype)
    check_lse(to_np(lse), rl, dtype)


def test_decode_is_independent_of_split_count():
    d = W.random_decode(31, [1500, 800, 3000], 16, 2, 128, 128)
    ro, rl = ref.decode(d.q, d.k, d.v, d.cu_seqlens_k, d.sink, d.softmax_scale)
    for splits in (1, 2, 5, 16, 47):
        out, lse = run_decode(d, splits)
        check_out(to_np(out), ro, "bf16", f"out[splits={splits}]")
        check_lse(to_np(lse), rl, "bf16", f"lse[splits={splits}]")
