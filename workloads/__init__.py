"""Seeded synthetic inputs for sink attention.

This module only draws inputs: random numbers, sequence lengths, packing offsets and
the bf16 rounding of the drawn values.  It holds none of the attention arithmetic, so
both the fp64 oracle (through the tests) and the CUDA path can be fed from it without
sharing any of the method's code.

Recipes (each config draws from ``numpy.random.default_rng(seed)`` in the order
written in its function: lengths first, then q, k, v, dout, sink):

* ``config1``  seed 0: 2 sequences of 256 tokens, 4 heads (q = kv), d = 64,
  sink ~ U(-2, 2), scale 1/8; the same data is run causal and non-causal.
* ``config2``  seed 1: 16 packed sequences, lengths ~ U[64, 4096] (inclusive),
  32 q heads / 8 kv heads, d = 128, causal, sink ~ N(0, 1), scale 1/sqrt(128).
* ``config3``  seed 2: 4 packed sequences of 8192 tokens, 16 heads, d = 128,
  causal, dout ~ N(0, 1), sink ~ N(0, 0.5) (0.5 read as the standard deviation).
* ``config4``  seed 3: 6 sequences, 1 head, 1024 queries against 1152 keys,
  dk = 64, dv = 32, bottom-right causal with window (512, 0), sink = log n.
* ``config5``  seed 4: decode, 64 sequences of one query each, key lengths
  ~ U[8192, 32768], 64 q heads / 8 kv heads, d = 128, sink ~ U(-1, 3).  Its 5 GB of
  K/V are drawn on the GPU with a seeded ``torch.Generator`` (``decode_kv_on_device``)
  and rounded to bf16 there; q, lengths and sink come from numpy.

Values are drawn as float32 and, for bf16 problems, rounded once to bf16 with
round-to-nearest-even; the rounded values are kept as float32 arrays whose every
element is exactly representable in bf16, so the GPU sees the same numbers the
oracle promotes to float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to the nearest bf16 (ties to even); returns float32.

    Works on the bit pattern in place: add 0x7FFF plus the lowest kept bit, then clear the
    16 dropped bits.  For finite inputs the sum cannot overflow 32 bits."""
    out = np.array(x, dtype=np.float32, copy=True, order="C")
    bits = out.view(np.uint32)
    lsb = bits >> 16
    lsb &= 1
    lsb += 0x7FFF
    bits += lsb
    bits &= np.uint32(0xFFFF0000)
    return out


@dataclass
class Problem:
    """One packed-THD sink-attention problem (host arrays)."""

    q: np.ndarray                    # [T_q, Hq, dk] float32 (bf16-exact when dtype == "bf16")
    k: np.ndarray                    # [T_k, Hkv, dk]
    v: np.ndarray                    # [T_k, Hkv, dv]
    cu_seqlens_q: np.ndarray         # [B + 1] int32
    cu_seqlens_k: np.ndarray         # [B + 1] int32
    sink: Optional[np.ndarray]       # [Hq] float32, may hold -inf; None = vanilla
    softmax_scale: float             # the float32 value handed to the kernels
    causal: bool = False
    window_left: int = -1
    window_right: int = -1
    dtype: str = "bf16"              # "bf16" or "fp32"
    dout: Optional[np.ndarray] = None  # [T_q, Hq, dv]
    name: str = ""
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.cu_seqlens_q.shape[0] - 1)

    @property
    def num_heads_q(self) -> int:
        return int(self.q.shape[1])

    @property
    def num_heads_kv(self) -> int:
        return int(self.k.shape[1])

    @property
    def head_dim_qk(self) -> int:
        return int(self.q.shape[2])

    @property
    def head_dim_v(self) -> int:
        return int(self.v.shape[2])

    @property
    def max_seqlen_q(self) -> int:
        return int(np.diff(self.cu_seqlens_q).max(initial=0))

    @property
    def max_seqlen_k(self) -> int:
        return int(np.diff(self.cu_seqlens_k).max(initial=0))


def _f32(x) -> float:
    return float(np.float32(x))


def cu_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    out = np.zeros(len(lengths) + 1, dtype=np.int32)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out


def fp16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest fp16 (ties to even, numpy's conversion); float32."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def _normal(rng, shape, std=1.0, dtype="bf16") -> np.ndarray:
    x = (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)
    if dtype == "bf16":
        return bf16_round(x)
    return fp16_round(x) if dtype == "fp16" else x


def _draw_sink(rng, hq: int, kind) -> Optional[np.ndarray]:
    if kind is None:
        return None
    if isinstance(kind, str):
        if kind == "normal":
            return rng.standard_normal(size=hq, dtype=np.float32)
        if kind == "uniform":
            return rng.uniform(-2.0, 2.0, size=hq).astype(np.float32)
        if kind == "neg_inf":
            return np.full(hq, -np.inf, dtype=np.float32)
        raise ValueError(f"unknown sink kind {kind!r}")
    arr = np.asarray(kind, dtype=np.float32)
    if arr.ndim == 0:
        arr = np.full(hq, float(arr), dtype=np.float32)
    assert arr.shape == (hq,)
    return arr


def random_problem(seed: int, lens_q: Sequence[int], lens_k: Sequence[int], hq: int, hkv: int,
                   dk: int, dv: int, causal: bool = False, window_left: int = -1,
                   window_right: int = -1, sink="normal", dtype: str = "bf16",
                   with_dout: bool = False, softmax_scale: Optional[float] = None,
                   name: str = "") -> Problem:
    """A small seeded problem for the parity tests (draw order: q, k, v, dout, sink)."""
    rng = np.random.default_rng(seed)
    cu_q = cu_from_lengths(lens_q)
    cu_k = cu_from_lengths(lens_k)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = _normal(rng, (tq, hq, dk), dtype=dtype)
    k = _normal(rng, (tk, hkv, dk), dtype=dtype)
    v = _normal(rng, (tk, hkv, dv), dtype=dtype)
    dout = _normal(rng, (tq, hq, dv), dtype=dtype) if with_dout else None
    s = _draw_sink(rng, hq, sink)
    scale = _f32(1.0 / math.sqrt(dk)) if softmax_scale is None else _f32(softmax_scale)
    return Problem(q, k, v, cu_q, cu_k, s, scale, causal, window_left, window_right, dtype,
                   dout, name or f"random_s{seed}")


# --- the five workload configurations ---------------------------------------------------

def config1(causal: bool) -> Problem:
    rng = np.random.default_rng(0)
    b, h, L, d = 2, 4, 256, 64
    cu = cu_from_lengths([L] * b)
    q = _normal(rng, (b * L, h, d))
    k = _normal(rng, (b * L, h, d))
    v = _normal(rng, (b * L, h, d))
    sink = rng.uniform(-2.0, 2.0, size=h).astype(np.float32)
    return Problem(q, k, v, cu, cu.copy(), sink, _f32(1.0 / 8.0), causal, -1, -1, "bf16",
                   None, "fixed256_d64_" + ("causal" if causal else "full"))


def config2_lengths() -> np.ndarray:
    rng = np.random.default_rng(1)
    return rng.integers(64, 4096, size=16, endpoint=True)


def config2(dtype: str = "bf16") -> Problem:
    """The headline workload; dtype "fp16" rounds the same draws to fp16 instead of bf16."""
    rng = np.random.default_rng(1)
    lengths = rng.integers(64, 4096, size=16, endpoint=True)
    cu = cu_from_lengths(lengths)
    t = int(cu[-1])
    q = _normal(rng, (t, 32, 128), dtype=dtype)
    k = _normal(rng, (t, 8, 128), dtype=dtype)
    v = _normal(rng, (t, 8, 128), dtype=dtype)
    sink = rng.standard_normal(size=32, dtype=np.float32)
    return Problem(q, k, v, cu, cu.copy(), sink, _f32(1.0 / math.sqrt(128)), True, -1, -1,
                   dtype, None, "varlen16_gqa32x8_d128_causal" + ("_fp16" if dtype == "fp16" else ""))


def config3(with_dout: bool = True) -> Problem:
    rng = np.random.default_rng(2)
    b, L, h, d = 4, 8192, 16, 128
    cu = cu_from_lengths([L] * b)
    t = b * L
    q = _normal(rng, (t, h, d))
    k = _normal(rng, (t, h, d))
    v = _normal(rng, (t, h, d))
    dout = _normal(rng, (t, h, d))
    sink = (rng.standard_normal(size=h, dtype=np.float32) * np.float32(0.5)).astype(np.float32)
    return Problem(q, k, v, cu, cu.copy(), sink, _f32(1.0 / math.sqrt(128)), True, -1, -1,
                   "bf16", dout if with_dout else None, "train4x8192_h16_d128_causal")


def config4(n: float) -> Problem:
    rng = np.random.default_rng(3)
    b, sq, sk, dk, dv = 6, 1024, 1152, 64, 32
    cu_q = cu_from_lengths([sq] * b)
    cu_k = cu_from_lengths([sk] * b)
    q = _normal(rng, (b * sq, 1, dk))
    k = _normal(rng, (b * sk, 1, dk))
    v = _normal(rng, (b * sk, 1, dv))
    sink = np.full(1, math.log(n), dtype=np.float32)
    return Problem(q, k, v, cu_q, cu_k, sink, _f32(1.0 / math.sqrt(dk)), True, 512, 0, "bf16",
                   None, f"softmax_n{n:g}_b6_1024x1152_dk64_dv32_win512")


@dataclass
class DecodeProblem:
    """Decode: one query per sequence, q [B, Hq, dk]; K/V packed THD with cu_seqlens_k."""

    q: np.ndarray
    cu_seqlens_k: np.ndarray
    sink: Optional[np.ndarray]
    softmax_scale: float
    num_heads_kv: int
    head_dim_v: int
    causal: bool = True
    window_left: int = -1
    window_right: int = -1
    k: Optional[np.ndarray] = None   # host K/V when small; None when drawn on device
    v: Optional[np.ndarray] = None
    dtype: str = "bf16"
    name: str = ""


def config5_meta() -> DecodeProblem:
    rng = np.random.default_rng(4)
    b, hq, hkv, d = 64, 64, 8, 128
    lengths = rng.integers(8192, 32768, size=b, endpoint=True)
    q = _normal(rng, (b, hq, d))
    sink = rng.uniform(-1.0, 3.0, size=hq).astype(np.float32)
    return DecodeProblem(q, cu_from_lengths(lengths), sink, _f32(1.0 / math.sqrt(d)), hkv, d,
                         True, -1, -1, None, None, "bf16", "decode64_gqa64x8_d128_L8k-32k")


def decode_kv_on_device(total_k: int, hkv: int, dk: int, dv: int, seed: int = 4,
                        device="cuda", chunk_tokens: int = 1 << 18):
    """Draw K then V ~ N(0,1) on the GPU with a seeded Philox generator, rounded to bf16."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for width in (dk, dv):
        t = torch.empty((total_k, hkv, width), dtype=torch.bfloat16, device=device)
        for s in range(0, total_k, chunk_tokens):
            e = min(total_k, s + chunk_tokens)
            t[s:e] = torch.randn((e - s, hkv, width), generator=g, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
        out.append(t)
    return out[0], out[1]


def paged_layout(seed: int, lens_k: Sequence[int], block_size: int, spare_blocks: int = 3,
                 spare_columns: int = 1):
    """A block table for sequences of lens_k keys: each sequence gets ceil(len / block_size)
    physical blocks, drawn as a seeded random permutation of all num_blocks ids (so no
    sequence's blocks are adjacent or in order); `spare_blocks` ids stay unused and every
    row has `spare_columns` extra entries (set to a valid, unused id).
    Returns (block_table int32 [B, max_blocks], num_blocks)."""
    rng = np.random.default_rng(seed)
    per = [-(-int(n) // block_size) for n in lens_k]
    num_blocks = sum(per) + spare_blocks
    perm = rng.permutation(num_blocks).astype(np.int32)
    table = np.full((len(per), max(per + [0]) + spare_columns), perm[-1], dtype=np.int32)
    i = 0
    for b, n in enumerate(per):
        table[b, :n] = perm[i:i + n]
        i += n
    return table, num_blocks


def paged_rows(cu_seqlens_k, block_table, block_size: int):
    """For every packed key row (sequence b, key t): its (block, row-in-block) in the cache."""
    cu = np.asarray(cu_seqlens_k, dtype=np.int64)
    blk, off = [], []
    for b in range(len(cu) - 1):
        t = np.arange(int(cu[b + 1] - cu[b]))
        blk.append(np.asarray(block_table)[b, t // block_size])
        off.append(t % block_size)
    return np.concatenate(blk).astype(np.int64), np.concatenate(off).astype(np.int64)


def to_paged(x, cu_seqlens_k, block_table, block_size: int, num_blocks: int):
    """Packed rows x [total, H, d] (numpy or torch) laid out as a block cache
    [num_blocks, block_size, H, d]; unused cache rows are zero."""
    blk, off = paged_rows(cu_seqlens_k, block_table, block_size)
    if isinstance(x, np.ndarray):
        cache = np.zeros((num_blocks, block_size) + x.shape[1:], dtype=x.dtype)
        cache[blk, off] = x
        return cache
    import torch
    cache = torch.zeros((num_blocks, block_size) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    cache[torch.from_numpy(blk).to(x.device), torch.from_numpy(off).to(x.device)] = x
    return cache


def random_decode(seed: int, lens_k: Sequence[int], hq: int, hkv: int, dk: int, dv: int,
                  causal: bool = True, window_left: int = -1, window_right: int = -1,
                  sink="normal", dtype: str = "bf16") -> DecodeProblem:
    """A small seeded decode problem with host K/V (draw order: q, k, v, sink)."""
    rng = np.random.default_rng(seed)
    b = len(lens_k)
    cu_k = cu_from_lengths(lens_k)
    tk = int(cu_k[-1])
    q = _normal(rng, (b, hq, dk), dtype=dtype)
    k = _normal(rng, (tk, hkv, dk), dtype=dtype)
    v = _normal(rng, (tk, hkv, dv), dtype=dtype)
    s = _draw_sink(rng, hq, sink)
    return DecodeProblem(q, cu_k, s, _f32(1.0 / math.sqrt(dk)), hkv, dv, causal, window_left,
                         window_right, k, v, dtype, f"decode_s{seed}")
