"""Failure detection on the GPU without a fault: the attention kernel's bounded pipeline wait,
run on an mbarrier that nothing arrives at with a short limit, gives up, reports
MLA_ERR_DEVICE_TIMEOUT through the status word, and leaves the context usable."""
import time

import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    mla.load_library()


def test_bounded_wait_gives_up_and_reports():
    lib = mla.load_library()
    assert mla.mla_prefill_device_status() == 0
    t0 = time.time()
    assert lib.mla_selftest_wait_timeout(50, None) == 0
    st = mla.mla_prefill_device_status()  # synchronises
    elapsed = time.time() - t0
    assert st == 9, mla.mla_status_string(st)
    assert 0.04 < elapsed < 5.0
    assert mla.mla_prefill_device_status() == 0  # the status word was cleared by the read
    # the context is still usable: a normal call runs and is clean
    wl = W.Workload("after_timeout", [40], [60], 2, 1, seed=3)
    x = W.make_inputs(wl, device="cuda:0")
    out = torch.zeros(40, 2, 128, dtype=torch.bfloat16, device="cuda:0")
    mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                    mla.MLA_MASK_CAUSAL, 2, 1, wl.qk_scale, out)
    assert mla.mla_prefill_device_status() == 0
    assert torch.isfinite(out.float()).all() and out.abs().sum() > 0


def test_selftest_rejects_bad_limits():
    lib = mla.load_library()
    assert lib.mla_selftest_wait_timeout(0, None) == 6
    assert lib.mla_selftest_wait_timeout(20000, None) == 6
