"""The allocation-free entry point ``mla_prefill_noalloc``.

Some callers cannot call cudaMalloc: serving engines that reserve nearly all
GPU memory for their own pool at start-up, and latency-critical callers that
must never stall on a driver allocation.  For them the library offers
``mla_prefill_noalloc``, whose scratch is a fixed 1 MiB static device array.
Its results must be bit-identical to ``mla_prefill``'s: the same kernels run on
the same inputs, only the scratch memory differs.

This file is collected last on purpose.  It must pass in a fresh process and
after every other test.
"""
import ctypes

import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
from helpers import compare, cpu_copy, oracle_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(lens_q, lens_k, H, G, dtype, seed):
    wl = W.Workload("noalloc", lens_q, lens_k, H, G, dtype=dtype, seed=seed)
    return wl, W.make_inputs(wl, device=DEV)


def _padded(x, lens_k, max_seq, G):
    """Packed K / K_rope / V as the page's padded [batch, max_seq, G*W] tensors (NaN past Lk_b)."""
    out = {}
    for key, w in (("k", 128), ("k_rope", 64), ("v", 128)):
        buf = torch.full((len(lens_k), max_seq, G * w), float("nan"), dtype=x[key].dtype, device=DEV)
        start = 0
        for b, L in enumerate(lens_k):
            buf[b, :L] = x[key][start:start + L].reshape(L, G * w)
            start += L
        out[key] = buf
    return out


def _call_noalloc(lib, x, mask, H, G, scale, out):
    """Through the C ABI directly (ctypes), no Python-side wrapper logic."""
    d = [mla.as_mla_tensor(t) for t in (x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"],
                                        x["kv_seqlen"], out)]
    return lib.mla_prefill_noalloc(*(ctypes.byref(t) for t in d[:7]), mask, H, G, scale,
                                   ctypes.byref(d[7]), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_mla_prefill_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    lib = mla.load_library()
    # Three different problems, so each call reuses the static scratch the one before filled:
    # causal GQA (bf16), a causal chunk over a cached prefix (fp16), and no mask over the padded
    # K/V layout with NaN padding.
    problems = [([300, 37, 129], [300, 37, 129], 8, 2, torch.bfloat16, 5, mla.MLA_MASK_CAUSAL, 0),
                ([64, 512], [1000, 512], 4, 4, torch.float16, 6, mla.MLA_MASK_CAUSAL, 0),
                ([100, 7, 260], [90, 200, 260], 4, 2, torch.bfloat16, 7, mla.MLA_MASK_NONE, 384)]
    refs, cases = [], []
    mla.set_split_tiles(0)  # the allocation-free path never splits: compare like with like
    try:
        for lq, lk, H, G, dtype, seed, mask, max_seq in problems:
            wl, x = _case(lq, lk, H, G, dtype, seed)
            if max_seq:
                x = dict(x, **_padded(x, lk, max_seq, G))
            ref = torch.empty(wl.t_q, H, 128, dtype=dtype, device=DEV)
            mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                            mask, H, G, wl.qk_scale, ref)
            refs.append(ref)
            cases.append((wl, x, mask))
    finally:
        mla.set_split_tiles(-1)
    assert mla.mla_prefill_device_status() == 0
    # One warm-up call first: the first call on a GPU does the one-time set-up (the array's device
    # address, the module's first use), which is not part of what the calls below must not do.
    wl, x, mask = cases[0]
    warm = torch.empty_like(refs[0])
    assert _call_noalloc(lib, x, mask, wl.head_num, wl.kv_head_num, wl.qk_scale, warm) == 0
    outs = [torch.full_like(r, 7.0) for r in refs]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for (wl, x, mask), out in zip(cases, outs):
        rc = _call_noalloc(lib, x, mask, wl.head_num, wl.kv_head_num, wl.qk_scale, out)
        assert rc == 0, mla.mla_status_string(rc)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, "device memory changed across allocation-free calls"
    assert mla.mla_prefill_device_status() == 0
    # the same kernels on the same inputs: bit for bit the result of mla_prefill
    assert torch.equal(warm, refs[0])
    for (wl, x, mask), out, ref in zip(cases, outs, refs):
        assert torch.equal(out, ref)
    # and against the fp64 oracle with the usual bound (the first problem)
    wl, x, mask = cases[0]
    ref = oracle_rows(cpu_copy(x), wl.head_num, wl.kv_head_num, wl.qk_scale)
    ok, st = compare(outs[0].cpu(), ref, wl.dtype)
    assert ok, st


def test_noalloc_reports_clamped_seqlens():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    lib = mla.load_library()
    wl, x = _case([100, 60], [100, 60], 2, 1, torch.bfloat16, 8)
    x["q_seqlen"] = torch.tensor([100, 90], dtype=torch.int32, device=DEV)  # sums past T_q = 160
    guard = 64
    buf = torch.full((160 + 2 * guard, 2, 128), 5.0, dtype=torch.bfloat16, device=DEV)
    out = buf[guard:guard + 160]
    assert mla.mla_prefill_device_status() == 0
    assert _call_noalloc(lib, x, mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out) == 0
    assert mla.mla_prefill_device_status() == 8  # MLA_ERR_SEQLEN, from the static array's word
    assert mla.mla_prefill_device_status() == 0  # reading clears it
    assert torch.all(buf[:guard] == 5.0) and torch.all(buf[guard + 160:] == 5.0)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = mla.load_library()
    # descriptors only: the size check happens on the host before any device access
    fake = 1 << 20  # an aligned address that is never dereferenced

    def desc(shape, dtype):
        t = mla.MlaTensor()
        t.data = fake
        t.dtype = dtype
        t.ndim = len(shape)
        stride = 1
        for i in reversed(range(len(shape))):
            t.shape[i] = shape[i]
            t.stride[i] = stride
            stride *= shape[i]
        return t

    T = 1 << 27  # 134M query tokens: the unit list alone needs far more than 1 MiB
    q, qr = desc((T, 1, 128), mla.MLA_BF16), desc((T, 1, 64), mla.MLA_BF16)
    k, kr, v = desc((16, 1, 128), mla.MLA_BF16), desc((16, 1, 64), mla.MLA_BF16), desc((16, 1, 128), mla.MLA_BF16)
    qs, ks = desc((1,), mla.MLA_I32), desc((1,), mla.MLA_I32)
    out = desc((T, 1, 128), mla.MLA_BF16)
    out.data = fake + (1 << 40)  # disjoint from the inputs
    rc = lib.mla_prefill_noalloc(ctypes.byref(q), ctypes.byref(qr), ctypes.byref(k), ctypes.byref(kr),
                                 ctypes.byref(v), ctypes.byref(qs), ctypes.byref(ks), mla.MLA_MASK_CAUSAL, 1, 1,
                                 0.1, ctypes.byref(out), None)
    assert rc == 6  # MLA_ERR_UNSUPPORTED
