"""Which attention kernel a call runs, as the header documents it (mla_prefill_set_kernel):
automatically the CTA-pair kernel for packed, unsplit K/V with long sequences (on average 3072 keys
or more per sequence) once its work units give at least one item per SM pair, else the single-CTA
kernel; forced choices; padded K/V and split-KV always on the single-CTA kernel.  The choice tests
run with split-KV off (it is chosen first, for problems with few items per SM); one test checks that
it takes precedence.  Each call is also checked against the fp64 oracle on sampled rows, so the
choice never trades correctness."""
import numpy as np
import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
from helpers import compare, cpu_copy, oracle_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SINGLE, PAIR = 1, 2


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mla.load_library()
    torch.cuda.set_device(0)
    yield
    mla.set_kernel(-1)
    torch.cuda.synchronize()


@pytest.fixture(autouse=True)
def no_split():
    mla.set_split_tiles(0)
    yield
    mla.set_split_tiles(-1)
    mla.set_kernel(-1)


def last_kernel():
    return mla.load_library().mla_prefill_last_kernel()


def run_and_check(lens_q, lens_k, H, G, seed, launches=2):
    wl = W.Workload("choice", list(lens_q), list(lens_k), H, G, seed=seed)
    x = W.make_inputs(wl, device=DEV)
    out = torch.full((wl.t_q, H, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                    mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, out)
    assert mla.mla_prefill_device_status() == 0
    kernel = last_kernel()
    assert mla.load_library().mla_prefill_last_launches() == launches  # plan + attention (+ combine)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, wl.t_q - 1], rng.choice(wl.t_q, 48, replace=False)]))
    ref = oracle_rows(cpu_copy(x), H, G, wl.qk_scale, rows=rows)
    ok, st = compare(out.cpu()[rows], ref[rows], torch.bfloat16)
    assert ok, st
    return kernel


def sm_count():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_automatic_choice_long_sequences_run_on_pairs():
    mla.set_kernel(-1)
    # 4096 keys per sequence; (4096 / 512 + 1) units x 32 heads >= one item per SM pair
    assert run_and_check([4096], [4096], 32, 32, seed=1) == PAIR
    # the same with four query heads per kv head (head-pair units: 4096 / 256 + 1 units x 16 pairs)
    assert run_and_check([4096], [4096], 32, 8, seed=2) == PAIR


def test_automatic_choice_short_sequences_run_on_single_ctas():
    mla.set_kernel(-1)
    assert run_and_check([1024] * 4, [1024] * 4, 16, 16, seed=3) == SINGLE   # 1024 keys per sequence
    assert run_and_check([2000, 300], [2000, 300], 8, 2, seed=4) == SINGLE   # 1150 on average


def test_automatic_choice_needs_enough_items_for_the_pairs():
    mla.set_kernel(-1)
    # long keys but too few items to give every SM pair one: (4096 / 512 + 1) units x 2 heads
    items = (4096 // 512 + 1) * 2
    assert items < sm_count() // 2
    assert run_and_check([4096], [4096], 2, 2, seed=5) == SINGLE


@pytest.mark.parametrize("forced", [SINGLE, PAIR])
def test_forced_choice_is_honoured(forced):
    mla.set_kernel(forced)
    try:
        assert run_and_check([600, 90], [600, 90], 4, 2, seed=10 + forced) == forced
        assert run_and_check([4096], [4096], 32, 32, seed=20 + forced) == forced
    finally:
        mla.set_kernel(-1)


def test_padded_kv_runs_on_single_ctas_even_when_pairs_are_forced():
    lens, H, G, max_seq = [700, 333], 4, 2, 768
    wl = W.Workload("padded", lens, lens, H, G, seed=31)
    x = W.make_inputs(wl, device=DEV)
    padded = {}
    for key, width in (("k", 128), ("k_rope", 64), ("v", 128)):
        buf = torch.zeros(len(lens), max_seq, G * width, dtype=torch.bfloat16, device=DEV)
        start = 0
        for b, L in enumerate(lens):
            buf[b, :L] = x[key][start:start + L].reshape(L, G * width)
            start += L
        padded[key] = buf
    out = torch.empty(wl.t_q, H, 128, dtype=torch.bfloat16, device=DEV)
    mla.set_kernel(PAIR)
    try:
        mla.mla_prefill(x["q"], x["q_rope"], padded["k"], padded["k_rope"], padded["v"], x["q_seqlen"],
                        x["kv_seqlen"], mla.MLA_MASK_CAUSAL, H, G, wl.qk_scale, out)
        assert mla.mla_prefill_device_status() == 0
        assert last_kernel() == SINGLE
    finally:
        mla.set_kernel(-1)
    rows = np.arange(0, wl.t_q, 37)
    ok, st = compare(out.cpu()[rows], oracle_rows(cpu_copy(x), H, G, wl.qk_scale, rows=rows)[rows], torch.bfloat16)
    assert ok, st


def test_split_kv_takes_precedence_and_runs_on_single_ctas():
    # one long sequence at 16 heads: too few items for the SMs, so the automatic split-KV chunks it,
    # and split-KV runs on the single-CTA kernel (plan + attention + combine), also with pairs forced
    mla.set_split_tiles(-1)
    for forced in (-1, PAIR):
        mla.set_kernel(forced)
        assert run_and_check([4096], [4096], 16, 16, seed=40, launches=3) == SINGLE
