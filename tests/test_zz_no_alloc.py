"""The allocation-free entry point ``mla_prefill_noalloc``.

Some callers cannot call cudaMalloc: serving engines that reserve nearly all
GPU memory for their own pool at start-up, and latency-critical callers that
must never stall on a driver allocation.  For them the library offers
``mla_prefill_noalloc``, whose scratch is a fixed 1 MiB static device array.

This file is collected last on purpose.  It must pass in a fresh process and
after every other test.
"""
import ctypes

import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
from helpers import compare

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(lens_q, lens_k, H, G, dtype, seed):
    wl = W.Workload("noalloc", lens_q, lens_k, H, G, dtype=dtype, seed=seed)
    return wl, W.make_inputs(wl, device=DEV)


def _call_noalloc(lib, x, H, G, scale, out):
    """Through the C ABI directly (ctypes), no Python-side wrapper logic."""
    d = [mla.as_mla_tensor(t) for t in (x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"],
                                        x["kv_seqlen"], out)]
    return lib.mla_prefill_noalloc(*(ctypes.byref(t) for t in d[:7]), mla.MLA_MASK_CAUSAL, H, G, scale,
                                   ctypes.byref(d[7]), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_mla_prefill_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    lib = mla.load_library()
    # two different problems, so the second call reuses the static scratch the first one filled
    problems = [([300, 37, 129], [300, 37, 129], 8, 2, torch.bfloat16, 5),
                ([64, 512], [1000, 512], 4, 4, torch.float16, 6)]
    refs, cases = [], []
    for lq, lk, H, G, dtype, seed in problems:
        wl, x = _case(lq, lk, H, G, dtype, seed)
        ref = torch.empty(wl.t_q, H, 128, dtype=dtype, device=DEV)
        mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                        mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, ref)
        refs.append(ref)
        cases.append((wl, x))
    outs = [torch.full_like(r, 7.0) for r in refs]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for (wl, x), out in zip(cases, outs):
        rc = _call_noalloc(lib, x, wl.head_num, wl.kv_head_num, wl.qk_scale, out)
        assert rc == 0, mla.mla_status_string(rc)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, "device memory changed across allocation-free calls"
    for (wl, x), out, ref in zip(cases, outs, refs):
        ok, st = compare(out.cpu(), ref.double().cpu().numpy(), wl.dtype)
        assert ok, st


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
