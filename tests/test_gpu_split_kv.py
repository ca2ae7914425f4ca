"""GPU parity of split-KV (mla_prefill_set_split_tiles): a unit's key tiles in chunks, each chunk
a work item with fp32 partial rows, merged by the combine kernel.  The result is the same
softmax over all keys, so every case is checked against the fp64 oracle with the usual bound
(tests/helpers.py), and against the unsplit kernel within a few output ulps."""
import numpy as np
import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
from helpers import compare, cpu_copy, oracle_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mla.load_library()
    torch.cuda.set_device(0)
    yield
    mla.set_split_tiles(-1)
    torch.cuda.synchronize()


def run(x, H, G, scale, mask, split, out=None):
    mla.set_split_tiles(split)
    try:
        if out is None:
            out = torch.full((x["q"].shape[0], H, 128), 7.0, dtype=x["q"].dtype, device=DEV)
        mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"], mask, H,
                        G, scale, out)
        torch.cuda.synchronize()
    finally:
        mla.set_split_tiles(-1)
    return out


def check(x, out, H, G, scale, mask, rows=None, head_chunk=None, bound="literal"):
    ref = oracle_rows(cpu_copy(x), H, G, scale, rows=rows,
                      mask_type=1 if mask == mla.MLA_MASK_CAUSAL else 0, head_chunk=head_chunk)
    computed = ~np.isnan(ref[:, 0, 0])
    ok, st = compare(out.cpu(), ref, x["q"].dtype, mask=computed, bound=bound)
    assert ok, st


CASES = [
    # lq, lk, H, G, dtype, mask, split tiles
    ([300, 1, 700], [300, 1, 700], 4, 2, torch.bfloat16, mla.MLA_MASK_CAUSAL, 1),
    ([300, 1, 700], [300, 1, 700], 4, 2, torch.bfloat16, mla.MLA_MASK_CAUSAL, 2),
    ([64, 200, 90], [900, 200, 40], 2, 2, torch.float16, mla.MLA_MASK_CAUSAL, 3),   # chunks; Lq > Lk rows
    ([129, 257], [1000, 513], 4, 1, torch.bfloat16, mla.MLA_MASK_NONE, 2),
    ([600], [600], 1, 1, torch.float16, mla.MLA_MASK_NONE, 1),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_split_against_oracle_and_unsplit(case):
    lq, lk, H, G, dtype, mask, split = CASES[case]
    wl = W.Workload("split_case", lq, lk, H, G, dtype=dtype, seed=800 + case)
    x = W.make_inputs(wl, device=DEV)
    whole = run(x, H, G, wl.qk_scale, mask, 0)
    assert mla.load_library().mla_prefill_last_launches() == 2  # plan + attention
    parts = run(x, H, G, wl.qk_scale, mask, split)
    assert mla.load_library().mla_prefill_last_launches() == 3  # + combine
    assert mla.mla_prefill_device_status() == 0
    check(x, parts, H, G, wl.qk_scale, mask)
    n = sum(lq)
    assert torch.all(parts[n:] == 7.0)  # rows past sum(q_seqlen) untouched
    # same softmax, different summation order: within a few output ulps of the unsplit kernel
    d = (parts[:n].float() - whole[:n].float()).abs()
    assert d.max().item() <= 4 * 2.0 ** -8 * max(1.0, whole[:n].float().abs().max().item())


def test_split_padded_and_paged_layouts():
    lq, lk, H, G = [100, 300], [500, 300], 4, 2
    wl = W.Workload("split_layouts", lq, lk, H, G, seed=811)
    x = W.make_inputs(wl, device=DEV)
    ref = run(x, H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL, 2)
    # padded [batch, max_seq, G*W], padding NaN
    pad = {}
    for key, w in (("k", 128), ("k_rope", 64), ("v", 128)):
        buf = torch.full((2, 512, G * w), float("nan"), dtype=torch.bfloat16, device=DEV)
        start = 0
        for b, L in enumerate(lk):
            buf[b, :L] = x[key][start:start + L].reshape(L, G * w)
            start += L
        pad[key] = buf
    got = run(dict(x, **pad), H, G, wl.qk_scale, mla.MLA_MASK_CAUSAL, 2)
    assert torch.equal(got, ref)
    # paged, block size 32, NaN in unused slots
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], lk, 32, seed=3, slot_fill=float("nan"))
    mla.set_split_tiles(2)
    try:
        out = torch.empty_like(ref)
        mla.mla_prefill_paged(x["q"], x["q_rope"], kc, vc, table, x["q_seqlen"], x["kv_seqlen"],
                              mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, out)
        torch.cuda.synchronize()
    finally:
        mla.set_split_tiles(-1)
    assert mla.mla_prefill_device_status() == 0
    assert torch.equal(out, ref)


def test_automatic_split_long_sequence_one_head():
    # one long sequence with one head: 65 units cannot fill the SMs, so the library splits
    wl = W.Workload("long_h1", [16384], [16384], 1, 1, seed=4)
    x = W.make_inputs(wl, device=DEV)
    auto = run(x, 1, 1, wl.qk_scale, mla.MLA_MASK_CAUSAL, -1)
    whole = run(x, 1, 1, wl.qk_scale, mla.MLA_MASK_CAUSAL, 0)
    assert mla.mla_prefill_device_status() == 0
    assert not torch.equal(auto, whole)  # the automatic path did split (different summation order)
    rows = W.sample_rows(16384, 48, seed=9)
    check(x, auto, 1, 1, wl.qk_scale, mla.MLA_MASK_CAUSAL, rows=rows)


def test_split_control_rejects_bad_values():
    with pytest.raises(mla.MlaError):
        mla.set_split_tiles(-2)


def test_one_tile_chunks_over_many_short_sequences():
    # every work item a single key tile: the pipeline turns over once per item; units of one key
    # tile are written directly, the others (up to nine chunks) merged by the combine kernel
    rng = np.random.default_rng(79)
    lens = [int(v) for v in rng.integers(1, 301, 300)] + [1100, 1024]
    lens = [lens[i] for i in rng.permutation(len(lens))]
    wl = W.Workload("split_many", lens, lens, 4, 2, seed=812)
    x = W.make_inputs(wl, device=DEV)
    whole = run(x, 4, 2, wl.qk_scale, mla.MLA_MASK_CAUSAL, 0)
    parts = run(x, 4, 2, wl.qk_scale, mla.MLA_MASK_CAUSAL, 1)
    assert mla.mla_prefill_device_status() == 0
    # Half-ulp form of the bound: 24M checked elements, most in rows with a handful of keys where
    # |out| reaches 2-4 and the bf16 storage rounding alone is up to 0.0078 (0.0156 above 4).
    check(x, parts, 4, 2, wl.qk_scale, mla.MLA_MASK_CAUSAL, bound="half_ulp")
    d = (parts.float() - whole.float()).abs()
    assert d.max().item() <= 4 * 2.0 ** -8 * max(1.0, whole.float().abs().max().item())
