"""GPU parity of mla_prefill_paged: attention reading K / K_rope / V in place from
block-paged caches through a block table.

Its result is defined as the PagedCacheLoadOperation gather (no seqStarts)
followed by the MLA Prefill attention, so every case checks it bit-exactly
against mla_prefill on the same keys in packed form (and against the gather ->
mla_prefill composition), plus directly against the fp64 oracle on small cases.
"""
import numpy as np
import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
from helpers import compare, cpu_copy, oracle_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
NAN = float("nan")


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mla.load_library()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def problem(lq, lk, H, G, dtype=torch.bfloat16, seed=0):
    wl = W.Workload("paged_case", list(lq), list(lk), H, G, dtype=dtype, seed=seed)
    return wl, W.make_inputs(wl, device=DEV)


def packed(x, H, G, scale, mask):
    """Packed K/V on the single-CTA kernel, the kernel paged K/V runs on (same key tiles): the paged
    result must match it bit for bit."""
    out = torch.full((x["q"].shape[0], H, 128), 7.0, dtype=x["q"].dtype, device=DEV)
    mla.set_kernel(1)
    try:
        mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"], mask, H, G,
                        scale, out)
    finally:
        mla.set_kernel(-1)
    return out


def paged(x, kc, vc, table, H, G, scale, mask, out=None):
    if out is None:
        out = torch.full((x["q"].shape[0], H, 128), 7.0, dtype=x["q"].dtype, device=DEV)
    mla.mla_prefill_paged(x["q"], x["q_rope"], kc, vc, table, x["q_seqlen"], x["kv_seqlen"], mask, H, G, scale, out)
    return out


def status():
    return mla.mla_prefill_device_status()


CASES = [
    # lq, lk, H, G, block_size, dtype, mask
    ([100, 1, 300], [100, 1, 300], 4, 2, 16, torch.bfloat16, mla.MLA_MASK_CAUSAL),
    ([64, 200, 5], [700, 200, 133], 8, 2, 64, torch.float16, mla.MLA_MASK_CAUSAL),
    ([129, 257], [1000, 257], 2, 1, 8, torch.bfloat16, mla.MLA_MASK_CAUSAL),
    ([90, 33], [600, 33], 2, 2, 32, torch.bfloat16, mla.MLA_MASK_NONE),
    ([300, 17], [900, 400], 4, 4, 128, torch.float16, mla.MLA_MASK_CAUSAL),
    ([40, 256, 1], [1100, 256, 640], 4, 1, 256, torch.bfloat16, mla.MLA_MASK_CAUSAL),
    ([77], [77], 1, 1, 512, torch.bfloat16, mla.MLA_MASK_NONE),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_paged_equals_packed_bit_exactly(case):
    lq, lk, H, G, bs, dtype, mask = CASES[case]
    wl, x = problem(lq, lk, H, G, dtype, seed=700 + case)
    ref = packed(x, H, G, wl.qk_scale, mask)
    # unused slots and table entries hold junk: NaN slots, block ids far out of range
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=case, spare_blocks=3, slot_fill=NAN,
                                  table_fill=1 << 30)
    out = paged(x, kc, vc, table, H, G, wl.qk_scale, mask)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)


def test_paged_against_oracle():
    lq, lk, H, G, bs = [60, 200, 1], [300, 200, 90], 4, 2, 16
    wl, x = problem(lq, lk, H, G, seed=720)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=3, slot_fill=-float("inf"))
    out = paged(x, kc, vc, table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    ref = oracle_rows(cpu_copy(x), H, G, wl.qk_scale)
    n = sum(lq)
    ok, st = compare(out[:n].cpu(), ref[:n], x["q"].dtype)
    assert ok, st
    assert torch.all(out[n:] == 7.0)  # rows past sum(q_seqlen) untouched


def test_paged_equals_gather_then_prefill():
    lq, lk, H, G, bs = [64, 200], [700, 200], 4, 2, 64
    wl, x = problem(lq, lk, H, G, seed=721)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=4, spare_blocks=2, slot_fill=NAN)
    key = torch.empty(wl.t_k, G, 192, dtype=x["k"].dtype, device=DEV)
    value = torch.empty(wl.t_k, G, 128, dtype=x["k"].dtype, device=DEV)
    mla.mla_paged_cache_load(kc, vc, table, x["kv_seqlen"], key, value)
    y = dict(x, k=key[:, :, :128], k_rope=key[:, :, 128:], v=value)
    ref = packed(y, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    out = paged(x, kc, vc, table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)


def test_strided_cache_views():
    # caches as views into wider per-slot buffers (head and slot strides > width)
    lq, lk, H, G, bs = [50, 130], [400, 130], 4, 2, 32
    wl, x = problem(lq, lk, H, G, seed=722)
    ref = packed(x, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=5)
    kw = torch.full(kc.shape[:3] + (256,), NAN, dtype=kc.dtype, device=DEV)
    kw[..., 64:256] = kc
    vw = torch.full(vc.shape[:2] + (G + 1, 128), NAN, dtype=vc.dtype, device=DEV)
    vw[:, :, 1:] = vc
    out = paged(x, kw[..., 64:256], vw[:, :, 1:], table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)


def test_out_of_range_block_of_a_visible_key_is_reported():
    lq, lk, H, G, bs = [40, 40], [200, 40], 2, 1, 16
    wl, x = problem(lq, lk, H, G, seed=723)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=6)
    table = table.clone()
    table[0, 3] = kc.shape[0] + 5
    out = paged(x, kc, vc, table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 10
    assert torch.isfinite(out[:80].float()).all()
    # the same result as the gather, which writes that block's keys as zeros
    key = torch.empty(wl.t_k, G, 192, dtype=x["k"].dtype, device=DEV)
    value = torch.empty(wl.t_k, G, 128, dtype=x["k"].dtype, device=DEV)
    mla.mla_paged_cache_load(kc, vc, table, x["kv_seqlen"], key, value)
    assert status() == 10
    y = dict(x, k=key[:, :, :128], k_rope=key[:, :, 128:], v=value)
    ref = packed(y, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_kv_longer_than_the_table_is_clamped_and_reported():
    lq, lk, H, G, bs = [30, 30], [64, 30], 2, 1, 16
    wl, x = problem(lq, lk, H, G, seed=724)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=7)
    assert table.shape[1] == 4
    y = dict(x, kv_seqlen=torch.tensor([90, 30], dtype=torch.int32, device=DEV))  # 90 > 4 * 16
    out = paged(y, kc, vc, table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 8
    assert torch.isfinite(out[:60].float()).all()


def test_empty_and_zero_length_sequences():
    lq, lk, H, G, bs = [0, 20, 5, 0], [0, 20, 0, 16], 2, 1, 8
    wl, x = problem(lq, lk, H, G, seed=725)
    ref = packed(x, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, bs, seed=8, slot_fill=NAN)
    out = paged(x, kc, vc, table, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)
    assert torch.all(out[20:25] == 0)  # rows with no visible key


def test_chunked_workload_sampled_rows():
    # the chunked-prefill workload (8 x 4096 cached keys, 128 heads) read from a 64-slot paged cache
    wl = W.get("chunked")
    x = W.make_inputs(wl, device=DEV)
    ref = packed(x, wl.head_num, wl.kv_head_num, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], wl.kv_seqlens, 64, seed=9)
    del x["k"], x["k_rope"], x["v"]
    out = paged(x, kc, vc, table, wl.head_num, wl.kv_head_num, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)


def test_many_short_sequences_paged_equals_packed():
    # many one- and two-tile units per CTA through the warp-wide paged producer
    rng = np.random.default_rng(78)
    lens = [int(v) for v in rng.integers(1, 301, 400)] + [1500, 2048]
    lens = [lens[i] for i in rng.permutation(len(lens))]
    wl, x = problem(lens, lens, 4, 2, torch.bfloat16, seed=7800)
    ref = packed(x, 4, 2, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lens, 32, seed=78, spare_blocks=5, slot_fill=NAN,
                                  table_fill=1 << 30)
    out = paged(x, kc, vc, table, 4, 2, wl.qk_scale, mla.MLA_MASK_CAUSAL)
    torch.cuda.synchronize()
    assert status() == 0
    assert torch.equal(out, ref)
