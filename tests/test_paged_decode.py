"""Paged-KV decode (CANN flash_attn doc, "Paged Attention Parameter Group"; PA_BBND K/V
layout) on the GPU against the oracle's paged decode: every output element on small
seeded problems with shuffled physical blocks, partly used tail blocks, shared blocks and
empty sequences; sampled rows of the full decode workload in paged form; and the device
status for table entries outside the cache."""
import numpy as np
import pytest

import workloads as W
from oracle import ref
from _check import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu

try:
    import torch
    import softmax_attn_sink_b200 as sab
except Exception:  # torch without CUDA still imports; the calls fail at run time
    pass


def _dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(dtype) if dtype is not None else t


def _run(d, table, used, bs, kc, vc, splits=0, max_k=None):
    mk = max_k if max_k is not None else max(int(np.max(used)), 1)
    out, lse = sab.attn_sink_decode_paged(
        _dev(d.q, torch.bfloat16), _dev(kc, torch.bfloat16), _dev(vc, torch.bfloat16),
        _dev(table), _dev(used), mk, None if d.sink is None else _dev(d.sink), d.softmax_scale,
        d.causal, (d.window_left, d.window_right), splits)
    torch.cuda.synchronize()
    return out, lse


PAGED_CASES = [
    # name, lens_k, hq, hkv, dk, dv, block_size, window_left, sink, splits
    ("bs16_gqa8", [1, 15, 16, 17, 300, 1000], 16, 2, 128, 128, 16, -1, "normal", 0),
    ("bs48_gqa4", [47, 48, 49, 777], 8, 2, 128, 128, 48, -1, "normal", 0),
    ("bs64_splits5", [640, 65, 0, 2000], 8, 1, 128, 128, 64, -1, "uniform", 5),
    ("bs256_window", [1000, 300], 8, 2, 128, 128, 256, 200, "normal", 3),
    ("bs1024_mha", [2100, 5], 4, 4, 128, 128, 1024, -1, "normal", 0),
    ("bs32_dk64_dv32", [333, 31, 64], 8, 2, 64, 32, 32, -1, "normal", 0),
    ("bs16_no_sink", [129, 250], 8, 2, 128, 64, 16, -1, None, 0),
    # one split over 70000 keys: 4377 block ids do not fit next to the pipeline in shared
    # memory, so the kernel reads the table from global memory
    ("bs16_splits1_global_table", [70000, 3], 8, 1, 128, 128, 16, -1, "normal", 1),
    # head dim 256: two pipeline stages, one CTA per SM
    ("d256_bs64_gqa4", [700, 65, 1], 8, 2, 256, 256, 64, -1, "normal", 0),
]


@pytest.mark.parametrize("case", PAGED_CASES, ids=[c[0] for c in PAGED_CASES])
def test_paged_decode_matches_oracle(case):
    name, lens, hq, hkv, dk, dv, bs, wl, sink, splits = case
    seed = sum(map(ord, name))
    d = W.random_decode(seed, lens, hq, hkv, dk, dv, True, wl, -1 if wl < 0 else 0, sink)
    table, nb = W.paged_layout(seed + 1, lens, bs)
    kc = W.to_paged(d.k, d.cu_seqlens_k, table, bs, nb)
    vc = W.to_paged(d.v, d.cu_seqlens_k, table, bs, nb)
    used = np.asarray(lens, np.int32)
    out, lse = _run(d, table, used, bs, kc, vc, splits)
    ro, rl = ref.decode_paged(d.q, kc, vc, table, used, bs, d.sink, d.softmax_scale, True, wl,
                              -1 if wl < 0 else 0)
    check_out(to_np(out), ro, "bf16")
    check_lse(to_np(lse), rl, "bf16")
    assert sab.device_status()[0] == 0


def test_paged_decode_fp16():
    """fp16 K/V through a shuffled 48-key table."""
    lens = [47, 700, 1300]
    d = W.random_decode(21, lens, 8, 2, 128, 128, dtype="fp16")
    table, nb = W.paged_layout(22, lens, 48)
    kc = W.to_paged(d.k, d.cu_seqlens_k, table, 48, nb)
    vc = W.to_paged(d.v, d.cu_seqlens_k, table, 48, nb)
    used = np.asarray(lens, np.int32)
    out, lse = sab.attn_sink_decode_paged(
        _dev(d.q, torch.float16), _dev(kc, torch.float16), _dev(vc, torch.float16), _dev(table),
        _dev(used), max(lens), _dev(d.sink), d.softmax_scale, True)
    torch.cuda.synchronize()
    ro, rl = ref.decode_paged(d.q, kc, vc, table, used, 48, d.sink, d.softmax_scale, True)
    check_out(to_np(out), ro, "fp16")
    check_lse(to_np(lse), rl, "fp16")


def test_paged_equals_packed_decode_bits():
    """The same keys read packed or through a shuffled block table give identical bits when
    the chunking is the same (one split)."""
    lens = [500, 77, 1300]
    d = W.random_decode(5, lens, 8, 2, 128, 128)
    table, nb = W.paged_layout(6, lens, 64)
    kc = W.to_paged(d.k, d.cu_seqlens_k, table, 64, nb)
    vc = W.to_paged(d.v, d.cu_seqlens_k, table, 64, nb)
    o1, l1 = _run(d, table, np.asarray(lens, np.int32), 64, kc, vc, 1)
    o2, l2 = sab.attn_sink_decode(_dev(d.q, torch.bfloat16), _dev(d.k, torch.bfloat16),
                                  _dev(d.v, torch.bfloat16), _dev(d.cu_seqlens_k), max(lens),
                                  _dev(d.sink), d.softmax_scale, True, (-1, -1), 1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_shared_blocks():
    """Two sequences that name the same physical blocks (a shared prefix) and the same query
    get the same result."""
    lens = [300, 300]
    d = W.random_decode(8, lens, 8, 2, 128, 128)
    d.q[1] = d.q[0]
    table, nb = W.paged_layout(9, [300], 32)
    table = np.concatenate([table, table], axis=0)
    kc = W.to_paged(d.k[:300], np.array([0, 300]), table[:1], 32, nb)
    vc = W.to_paged(d.v[:300], np.array([0, 300]), table[:1], 32, nb)
    out, lse = _run(d, table, np.asarray(lens, np.int32), 32, kc, vc)
    o = to_np(out)
    assert np.array_equal(o[0], o[1])
    ro, rl = ref.decode_paged(d.q, kc, vc, table, np.asarray(lens, np.int32), 32, d.sink,
                              d.softmax_scale, True)
    check_out(o, ro, "bf16")
    check_lse(to_np(lse), rl, "bf16")


def test_bad_block_id_and_length_set_status():
    """A block id outside [0, num_blocks) and a key count beyond the table row are not read:
    the kernel skips them and the device status reports ATTN_SINK_ERR_BAD_INDEX (6)."""
    lens = [100, 100]
    d = W.random_decode(10, lens, 8, 2, 128, 128)
    table, nb = W.paged_layout(11, lens, 16)
    kc = W.to_paged(d.k, d.cu_seqlens_k, table, 16, nb)
    vc = W.to_paged(d.v, d.cu_seqlens_k, table, 16, nb)
    sab.device_status()   # clear
    bad = table.copy()
    bad[0, 2] = nb        # one past the last block
    out, _ = _run(d, bad, np.asarray(lens, np.int32), 16, kc, vc)
    assert sab.device_status()[0] == 6
    assert torch.isfinite(out.float()).all()
    too_long = np.asarray([table.shape[1] * 16 + 1, 100], np.int32)
    out, _ = _run(d, table, too_long, 16, kc, vc, max_k=int(too_long.max()))
    assert sab.device_status()[0] == 6
    # the context stays usable and a correct call is clean again
    out, lse = _run(d, table, np.asarray(lens, np.int32), 16, kc, vc)
    assert sab.device_status()[0] == 0
    ro, rl = ref.decode_paged(d.q, kc, vc, table, np.asarray(lens, np.int32), 16, d.sink,
                              d.softmax_scale, True)
    check_out(to_np(out), ro, "bf16")


def test_paged_config5_sampled():
    """The full decode workload (64 sequences of 8k-32k keys, 64/8 heads, d 128) through a
    shuffled 64-key block table, checked on sampled (sequence, kv head) rows."""
    d = W.config5_meta()
    lens = np.diff(d.cu_seqlens_k)
    total_k = int(d.cu_seqlens_k[-1])
    k, v = W.decode_kv_on_device(total_k, 8, 128, 128, seed=4)
    table, nb = W.paged_layout(40, lens, 64)
    kc = W.to_paged(k, d.cu_seqlens_k, table, 64, nb)
    vc = W.to_paged(v, d.cu_seqlens_k, table, 64, nb)
    out, lse = sab.attn_sink_decode_paged(_dev(d.q, torch.bfloat16), kc, vc, _dev(table),
                                          _dev(lens.astype(np.int32)), int(lens.max()),
                                          _dev(d.sink), d.softmax_scale, True)
    torch.cuda.synchronize()
    o, l = to_np(out), to_np(lse)
    rng = np.random.default_rng(103)
    for b in sorted(set([0, 63] + list(rng.integers(0, 64, size=3)))):
        k0, k1 = int(d.cu_seqlens_k[b]), int(d.cu_seqlens_k[b + 1])
        g = int(rng.integers(0, 8))
        kh = k[k0:k1, g].float().cpu().numpy()[:, None, :]
        vh = v[k0:k1, g].float().cpu().numpy()[:, None, :]
        heads = list(range(g * 8, g * 8 + 8))
        ro, rl = ref.decode(d.q[b:b + 1, heads], kh, vh, np.array([0, k1 - k0]), d.sink[heads],
                            d.softmax_scale)
        check_out(o[b, heads], ro[0], "bf16", f"out[b={b},g={g}]")
        check_lse(l[heads, b], rl[:, 0], "bf16", f"lse[b={b},g={g}]")
    assert sab.device_status()[0] == 0
