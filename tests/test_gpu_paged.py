"""GPU parity of the paged KV-cache gather (mla_paged_cache_load) against the
oracle in oracle/paged.py: byte work, so every comparison is bit-exact."""
import numpy as np
import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
import oracle.paged as paged

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mla.load_library()
    torch.cuda.set_device(0)


def _bits(t):
    """Host numpy view of the raw element bits (bf16 has no numpy dtype)."""
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy()
    return t.numpy()


def _random_cache(gen, nb, bs, H, D, dtype):
    if dtype == torch.int8:
        return torch.randint(-128, 127, (nb, bs, H, D), generator=gen, dtype=torch.int8).to(DEV)
    return torch.randn(nb, bs, H, D, generator=gen).to(dtype).to(DEV)


def make_case(seed, lens, bs, H, Dk, Dv, dtype, starts=None, extra_rows=3, spare_blocks=5):
    gen = torch.Generator().manual_seed(seed)
    need = [((0 if starts is None else s) + L + bs - 1) // bs for L, s in zip(lens, starts or [0] * len(lens))]
    width = max(need + [1])
    nb = sum(need) + spare_blocks
    kc = _random_cache(gen, nb, bs, H, Dk, dtype)
    vc = _random_cache(gen, nb, bs, H, Dv, dtype)
    perm = torch.randperm(nb, generator=gen)
    table = torch.full((len(lens), width), -1, dtype=torch.int32)
    used = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[used:used + n].to(torch.int32)
        used += n
    T = sum(lens) + extra_rows
    return kc, vc, table.to(DEV), T


def run(kc, vc, table, lens_t, T, starts=None, cumsum=False, fill=0x55):
    H, Dk, Dv = kc.shape[2], kc.shape[3], vc.shape[3]
    key = torch.full((T, H, Dk), fill, dtype=torch.int8, device=DEV).view(kc.dtype) if kc.dtype == torch.int8 \
        else torch.full((T, H, Dk), 3.0, dtype=kc.dtype, device=DEV)
    value = torch.full((T, H, Dv), fill, dtype=torch.int8, device=DEV).view(vc.dtype) if vc.dtype == torch.int8 \
        else torch.full((T, H, Dv), 3.0, dtype=vc.dtype, device=DEV)
    sentinel_k, sentinel_v = key.clone(), value.clone()
    mla.mla_paged_cache_load(kc, vc, table, lens_t, key, value, seq_starts=starts, cumsum=cumsum)
    torch.cuda.synchronize()
    return key, value, sentinel_k, sentinel_v


CASES = [
    # lens, block_size, H, Dk, Dv, dtype, with starts, cumsum
    ([300, 1, 129, 0, 64], 16, 2, 192, 128, torch.bfloat16, False, False),
    ([100, 257, 31], 64, 1, 576, 512, torch.float16, True, False),
    ([512, 513], 128, 4, 192, 128, torch.bfloat16, False, True),
    ([77, 5, 900], 32, 1, 512, 512, torch.int8, True, True),
    ([1], 1, 1, 8, 16, torch.bfloat16, False, False),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_paged_gather_bit_exact(case):
    lens, bs, H, Dk, Dv, dtype, with_starts, cumsum = CASES[case]
    starts = [((7 * b + 3) % (2 * bs)) for b in range(len(lens))] if with_starts else None
    kc, vc, table, T = make_case(40 + case, lens, bs, H, Dk, Dv, dtype, starts)
    ctx = np.concatenate([[11], 11 + np.cumsum(lens)]) if cumsum else np.array(lens)
    lens_t = torch.tensor(ctx, dtype=torch.int32, device=DEV)
    starts_t = torch.tensor(starts, dtype=torch.int32, device=DEV) if starts is not None else None
    key, value, sk, sv = run(kc, vc, table, lens_t, T, starts=starts_t, cumsum=cumsum)
    assert mla.mla_prefill_device_status() == 0
    rk, rv, bad = paged.paged_cache_load(_bits(kc), _bits(vc), table.cpu().numpy(), ctx, starts, cumsum)
    assert not bad
    n = sum(lens)
    assert np.array_equal(_bits(key)[:n], rk) and np.array_equal(_bits(value)[:n], rv)
    # rows past the total are untouched
    assert torch.equal(key[n:], sk[n:]) and torch.equal(value[n:], sv[n:])


def test_out_of_range_blocks_are_zeroed_and_reported():
    lens, bs = [40, 40], 16
    kc, vc, table, T = make_case(90, lens, bs, 2, 64, 64, torch.bfloat16)
    table = table.clone()
    table[0, 1] = kc.shape[0] + 3  # a block id past the cache
    table[1, 0] = -2               # a negative block id
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    key, value, _, _ = run(kc, vc, table, lens_t, T)
    assert mla.mla_prefill_device_status() == 10
    rk, rv, bad = paged.paged_cache_load(_bits(kc), _bits(vc), table.cpu().numpy(), lens)
    n = sum(lens)
    assert np.array_equal(_bits(key)[:n], rk) and np.array_equal(_bits(value)[:n], rv)
    assert sorted(bad) == list(range(16, 32)) + list(range(40, 56))


def test_lengths_past_the_output_are_clamped_and_reported():
    lens, bs = [50, 60], 16
    kc, vc, table, _ = make_case(91, lens, bs, 1, 64, 64, torch.float16)
    T = 70  # fewer rows than the 110 requested
    guard = 8
    key_buf = torch.full((T + guard, 1, 64), 5.0, dtype=torch.float16, device=DEV)
    val_buf = torch.full((T + guard, 1, 64), 5.0, dtype=torch.float16, device=DEV)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    mla.mla_paged_cache_load(kc, vc, table, lens_t, key_buf[:T], val_buf[:T])
    assert mla.mla_prefill_device_status() == 8
    assert torch.all(key_buf[T:] == 5.0) and torch.all(val_buf[T:] == 5.0)
    rk, _, _ = paged.paged_cache_load(_bits(kc), _bits(vc), table.cpu().numpy(), lens, num_tokens=T)
    assert np.array_equal(_bits(key_buf[:T]), rk)


def test_paged_gather_feeds_prefill_bit_identically():
    """Chunked prefill over a paged prefix: gather K (nope | rope = 192 columns) and V,
    then mla_prefill on the views equals mla_prefill on the original packed tensors."""
    lq, lk, H, G, bs = [64, 200], [700, 200], 4, 2, 64
    wl = W.Workload("paged", lq, lk, H, G, seed=92)
    x = W.make_inputs(wl, device=DEV)
    ref = torch.empty(wl.t_q, H, 128, dtype=torch.bfloat16, device=DEV)
    mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                    mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, ref)
    # scatter the packed K/V into a paged cache with a shuffled block table
    kcat = torch.cat([x["k"], x["k_rope"]], dim=2)  # [T_k, G, 192]
    need = [(L + bs - 1) // bs for L in lk]
    nb = sum(need) + 4
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(5))
    kc = torch.zeros(nb, bs, G, 192, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros(nb, bs, G, 128, dtype=torch.bfloat16, device=DEV)
    table = torch.full((len(lk), max(need)), -1, dtype=torch.int32)
    used, start = 0, 0
    for b, L in enumerate(lk):
        for i in range(need[b]):
            blk = int(perm[used + i])
            table[b, i] = blk
            n = min(bs, L - i * bs)
            kc[blk, :n] = kcat[start + i * bs:start + i * bs + n]
            vc[blk, :n] = x["v"][start + i * bs:start + i * bs + n]
        used += need[b]
        start += L
    key = torch.empty(wl.t_k, G, 192, dtype=torch.bfloat16, device=DEV)
    value = torch.empty(wl.t_k, G, 128, dtype=torch.bfloat16, device=DEV)
    mla.mla_paged_cache_load(kc, vc, table.to(DEV), x["kv_seqlen"], key, value)
    out = torch.empty_like(ref)
    mla.mla_prefill(x["q"], x["q_rope"], key[:, :, :128], key[:, :, 128:], value, x["q_seqlen"], x["kv_seqlen"],
                    mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, out)
    torch.cuda.synchronize()
    assert mla.mla_prefill_device_status() == 0
    assert torch.equal(out, ref)
