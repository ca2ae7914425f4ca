"""GPU checks of the caller-owned workspace path (mla_prefill_get_workspace_size + mla_prefill_ws),
the two phases of the MLA Prefill page's API (AtbMLAPreFillGetWorkspaceSize, then AtbMLAPreFill in
the caller's workspace).  The same kernels as mla_prefill run on the caller's memory, so results
must be bit-identical to mla_prefill's; with separate workspaces, calls on two streams may overlap."""
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


def _args(x):
    return (x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"])


def _workspace(x, H, G, scale, out, fill=0xA5):
    n = mla.mla_prefill_get_workspace_size(*_args(x), mla.MLA_MASK_CAUSAL, H, G, scale, out)
    ws = torch.full((n,), fill, dtype=torch.uint8, device=DEV)  # previous contents must not matter
    assert ws.data_ptr() % 256 == 0
    return ws


def test_two_streams_with_separate_workspaces():
    cases = [W.Workload("ws_a", [700, 90, 1300], [700, 90, 1300], 8, 2, seed=901),
             W.Workload("ws_b", [300, 512], [2000, 512], 16, 16, dtype=torch.float16, seed=902)]
    xs = [W.make_inputs(wl, device=DEV) for wl in cases]
    outs = [torch.full((wl.t_q, wl.head_num, 128), 7.0, dtype=wl.dtype, device=DEV) for wl in cases]
    wss = [_workspace(x, wl.head_num, wl.kv_head_num, wl.qk_scale, o) for wl, x, o in zip(cases, xs, outs)]
    refs = []
    for wl, x in zip(cases, xs):
        r = torch.empty(wl.t_q, wl.head_num, 128, dtype=wl.dtype, device=DEV)
        mla.mla_prefill(*_args(x), mla.MLA_MASK_CAUSAL, wl.head_num, wl.kv_head_num, wl.qk_scale, r)
        refs.append(r)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(3):  # several rounds, both streams in flight at once
        for wl, x, o, ws, s in zip(cases, xs, outs, wss, streams):
            with torch.cuda.stream(s):
                mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, wl.head_num, wl.kv_head_num, wl.qk_scale, o, ws,
                                   stream=s)
    for ws, s in zip(wss, streams):
        assert mla.mla_prefill_ws_status(ws, stream=s) == 0
    torch.cuda.synchronize()
    for wl, x, o, r in zip(cases, xs, outs, refs):
        assert torch.equal(o, r)  # same kernels, same inputs: bit-identical to mla_prefill
        ref = oracle_rows(cpu_copy(x), wl.head_num, wl.kv_head_num, wl.qk_scale)
        ok, st = compare(o.cpu(), ref, wl.dtype)
        assert ok, st
        print(wl.name, st)


def test_workspace_call_allocates_nothing():
    wl = W.Workload("ws_c", [333, 64], [333, 64], 4, 4, seed=903)
    x = W.make_inputs(wl, device=DEV)
    out = torch.empty(wl.t_q, 4, 128, dtype=wl.dtype, device=DEV)
    ws = _workspace(x, 4, 4, wl.qk_scale, out)
    mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, 4, 4, wl.qk_scale, out, ws)  # warm-up: module set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, 4, 4, wl.qk_scale, out, ws)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert mla.mla_prefill_ws_status(ws) == 0


def test_split_kv_in_the_caller_workspace():
    wl = W.Workload("ws_split", [1500, 100], [1500, 700], 2, 1, seed=904)
    x = W.make_inputs(wl, device=DEV)
    out = torch.full((wl.t_q, 2, 128), 7.0, dtype=wl.dtype, device=DEV)
    mla.set_split_tiles(2)
    try:
        n_split = mla.mla_prefill_get_workspace_size(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out)
        ws = _workspace(x, 2, 1, wl.qk_scale, out)
        mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out, ws)
        assert mla.load_library().mla_prefill_last_launches() == 3  # plan + attention + combine
        ref = torch.empty_like(out)
        mla.mla_prefill(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, ref)
        mla.set_split_tiles(0)
        n_plain = mla.mla_prefill_get_workspace_size(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out)
    finally:
        mla.set_split_tiles(-1)
    assert n_split > n_plain  # the fp32 partial rows live in the workspace too
    assert mla.mla_prefill_ws_status(ws) == 0
    assert torch.equal(out, ref)
    oracle_ref = oracle_rows(cpu_copy(x), 2, 1, wl.qk_scale)
    ok, st = compare(out.cpu(), oracle_ref, wl.dtype)
    assert ok, st


def test_status_is_per_call_and_too_small_is_rejected():
    wl = W.Workload("ws_bad", [100, 60], [100, 60], 2, 1, seed=905)
    x = W.make_inputs(wl, device=DEV)
    out = torch.full((160, 2, 128), 5.0, dtype=wl.dtype, device=DEV)
    ws = _workspace(x, 2, 1, wl.qk_scale, out, fill=0)
    bad = dict(x, q_seqlen=torch.tensor([100, 90], dtype=torch.int32, device=DEV))  # sums past T_q
    mla.mla_prefill_ws(*_args(bad), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out, ws)
    assert mla.mla_prefill_ws_status(ws) == 8  # MLA_ERR_SEQLEN, clamped
    mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out, ws)
    assert mla.mla_prefill_ws_status(ws) == 0  # the next call starts from 0
    assert mla.mla_prefill_device_status() == 0  # the library's own word saw nothing
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_ws(*_args(x), mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out, ws[:ws.numel() - 1])
    assert e.value.code == 11  # MLA_ERR_WORKSPACE
