"""GPU parity of mla_prolog (MLA Prolog, non-quantised) against the fp64 oracle in oracle/prolog.py.

Parity bounds, derived from the arithmetic of the CUDA path.  The projections
accumulate bf16 products in fp32 (relative error ~1e-6 at these depths); the
norms and the rotation run in fp32 with the library's rsqrtf (~2 ulp); outputs
are bf16, so an exactly computed value still carries half an ulp (subtracted
below as ulp_bf16(oracle) / 2).  The one rounding inside the chain is c^Q ->
bf16, a rounding decision the oracle takes in fp64 and the GPU in fp32: where
the two values straddle a bf16 midpoint (measured: ~0.2 % of c^Q elements at
the page's sizes) c^Q differs by one bf16 ulp, and each such element moves the
q elements of its row by ulp(c_i) |wq_b[i, j]| <= 2^-5 * 0.16 ~ 0.005 (|c| < 8,
|w| < 5 sigma).  Hence, per element (outputs have RMS ~1 by construction):
  * c^Q: equal to the oracle's except for < 1 % one-ulp flips, plus, for values
    near zero whose ulp is below the fp32 accumulation error of the projection
    (|gamma| sqrt(h) 2^-23 ~ 2e-5 at h = 4096), an absolute 2^-16;
  * q from the GPU's own c^Q (oracle.prolog.mla_prolog_q): excess <= 2^-12;
  * kv: excess <= 2^-12;
  * q through the whole chain: excess <= 2^-6 (a few flips per row at most).
"""
import numpy as np
import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import workloads as W
import oracle.prolog as prolog
from helpers import half_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIGHT = 2.0 ** -12
CHAIN = 2.0 ** -6
ORDER = ("token_x", "wq_a", "wq_b", "wkv", "rope_cos", "rope_sin", "gamma_cq", "gamma_ckv")


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mla.load_library()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def run(x, s, cq=True, q_out=None, kv_out=None):
    t = x["token_x"].shape[0]
    q = q_out if q_out is not None else torch.full((t, s.num_heads, s.head_dim), 7.0, dtype=torch.bfloat16,
                                                   device=DEV)
    kv = kv_out if kv_out is not None else torch.full((t, s.head_dim), 7.0, dtype=torch.bfloat16, device=DEV)
    c = torch.full((t, s.q_lora_rank), 7.0, dtype=torch.bfloat16, device=DEV) if cq else None
    mla.mla_prolog(*[x[k] for k in ORDER], s.num_heads, q, kv, c)
    torch.cuda.synchronize()
    return q, kv, c


def oracle_rows(x, s, rows):
    """The oracle on a subset of token rows (every step is per token)."""
    cpu = {k: v.cpu() for k, v in x.items()}
    for k in ("token_x", "rope_cos", "rope_sin"):
        cpu[k] = cpu[k][rows]
    return prolog.mla_prolog(*[cpu[k] for k in ORDER], s.num_heads)


def check(got, ref, bound):
    g = got.detach().float().cpu().double().numpy()
    assert np.all(np.isfinite(g))
    excess = np.abs(g - ref) - half_ulp(ref, torch.bfloat16)
    assert excess.max() <= bound, "max excess %.3g (max |err| %.3g)" % (excess.max(), np.abs(g - ref).max())
    return float(np.abs(g - ref).max())


def check_cq(got, ref):
    g = got.detach().float().cpu().double().numpy()
    diff = g != ref
    assert diff.mean() < 1e-2, "c^Q differs in %d of %d elements" % (diff.sum(), diff.size)
    if diff.any():  # a tie flip moves one bf16 ulp; near zero, fp32 accumulation error dominates the ulp
        assert np.all(np.abs(g - ref)[diff] <= 2 * half_ulp(ref[diff], torch.bfloat16) + 2.0 ** -16)


def check_all(x, s, rows, q, kv, cq):
    """c^Q, q from the GPU's c^Q, kv, and q through the whole chain, on the given token rows."""
    rq, rkv, rcq = oracle_rows(x, s, rows)
    check_cq(cq[rows], rcq)
    cpu = {k: v.cpu() for k, v in x.items()}
    rq_half = prolog.mla_prolog_q(cq[rows].cpu(), cpu["wq_b"], cpu["rope_cos"][rows], cpu["rope_sin"][rows],
                                  s.num_heads)
    check(q[rows], rq_half, TIGHT)
    check(kv[rows], rkv, TIGHT)
    check(q[rows], rq, CHAIN)


def test_small_full_against_oracle():
    s = W.prolog_shapes()["prolog_small"]
    x = W.make_prolog_inputs(s, device=DEV)
    q, kv, cq = run(x, s)
    assert mla.prolog_last_fused()  # head_dim 256, q_lora_rank 256: the fused q kernel
    check_all(x, s, np.arange(s.tokens), q, kv, cq)


def test_library_q_path_against_oracle_and_fused():
    # the same problem with the q projection forced onto the library GEMM + row kernel
    s = W.prolog_shapes()["prolog_small"]
    x = W.make_prolog_inputs(s, device=DEV)
    fq, fkv, fcq = run(x, s)
    mla.set_prolog_path(0)
    try:
        q, kv, cq = run(x, s)
        assert not mla.prolog_last_fused()
    finally:
        mla.set_prolog_path(-1)
    check_all(x, s, np.arange(s.tokens), q, kv, cq)
    assert torch.equal(cq, fcq) and torch.equal(kv, fkv)  # only the q projection differs
    # two fp32 accumulation orders of the same products, each rounded once to bf16: at most one ulp apart
    d = (q.float() - fq.float()).abs()
    assert torch.all(d <= 2 * torch.from_numpy(half_ulp(fq.float().cpu().double().numpy(), torch.bfloat16)).to(DEV)
                     + 2.0 ** -20)


@pytest.mark.parametrize("shape", [
    # head_dim 384: three N = 128 chunks per k-step; a ragged last tile of tokens
    dict(tokens=300, hidden=256, q_lora_rank=192, num_heads=3, head_dim=384, rope_dim=64, seed=65),
    # head_dim 128 with rope over all of it: both halves of the epilogue rotate
    dict(tokens=130, hidden=128, q_lora_rank=64, num_heads=2, head_dim=128, rope_dim=128, seed=66),
])
def test_fused_kernel_shapes(shape):
    s = W.PrologShape("prolog_fused", **shape)
    x = W.make_prolog_inputs(s, device=DEV, positions=np.random.default_rng(shape["seed"]).integers(0, 4096,
                                                                                                    s.tokens))
    q, kv, cq = run(x, s)
    assert mla.prolog_last_fused()
    check_all(x, s, np.arange(s.tokens), q, kv, cq)


def test_page_configuration_sampled_tokens():
    # the page's sizes: h 4096, q_lora_rank 1024, 64 heads of 512, rope 64; 4096 tokens
    s = W.prolog_shapes()["prolog"]
    x = W.make_prolog_inputs(s, device=DEV)
    q, kv, cq = run(x, s)
    assert mla.prolog_last_fused()
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4094, 4095],
                                     np.random.default_rng(5).choice(s.tokens, 25, replace=False)]))
    check_all(x, s, rows, q, kv, cq)


def test_tokens_across_the_internal_slab():
    # more tokens than one internal pass (4096): rows on both sides of the boundary and the tail
    s = W.PrologShape("prolog_slab", tokens=4096 + 37, hidden=256, q_lora_rank=128, num_heads=2, head_dim=128,
                      rope_dim=32, seed=62)
    x = W.make_prolog_inputs(s, device=DEV, positions=np.random.default_rng(1).integers(0, 65536, s.tokens))
    q, kv, cq = run(x, s)
    check_all(x, s, np.array([0, 4094, 4095, 4096, 4097, 4120, 4132]), q, kv, cq)


def test_single_token_and_without_cq_output():
    s = W.PrologShape("prolog_one", tokens=1, hidden=512, q_lora_rank=256, num_heads=3, head_dim=64, rope_dim=64,
                      seed=63)
    x = W.make_prolog_inputs(s, device=DEV, positions=[12345])
    q, kv, cq = run(x, s)
    check_all(x, s, np.arange(1), q, kv, cq)
    q2, kv2, _ = run(x, s, cq=False)
    assert torch.equal(q, q2) and torch.equal(kv, kv2)  # c^Q in library scratch: same result


def test_strided_views_and_guards():
    s = W.prolog_shapes()["prolog_small"]
    x = W.make_prolog_inputs(s, device=DEV)
    t, H, d = s.tokens, s.num_heads, s.head_dim
    ref_q, ref_kv, _ = run(x, s)
    # token_x with a wider row stride; q_out / kv_out as views into wider buffers
    xw = torch.zeros(t, s.hidden + 64, dtype=torch.bfloat16, device=DEV)
    xw[:, :s.hidden] = x["token_x"]
    qbuf = torch.full((t, H, d + 64), 5.0, dtype=torch.bfloat16, device=DEV)
    kvbuf = torch.full((t, d + 32), 5.0, dtype=torch.bfloat16, device=DEV)
    y = dict(x, token_x=xw[:, :s.hidden])
    q, kv, _ = run(y, s, q_out=qbuf[:, :, :d], kv_out=kvbuf[:, :d])
    assert torch.equal(q, ref_q) and torch.equal(kv, ref_kv)
    assert torch.all(qbuf[:, :, d:] == 5.0) and torch.all(kvbuf[:, d:] == 5.0)
    # q rows on 16-byte but not 32-byte boundaries (the fused epilogue's TMA store of a strided view)
    qbuf16 = torch.full((t, H, d + 16), 5.0, dtype=torch.bfloat16, device=DEV)
    q16 = qbuf16[:, :, 8:8 + d]
    assert q16.data_ptr() % 32 == 16
    run(x, s, q_out=q16)
    assert mla.prolog_last_fused()
    assert torch.equal(q16, ref_q)
    assert torch.all(qbuf16[:, :, :8] == 5.0) and torch.all(qbuf16[:, :, 8 + d:] == 5.0)
    # q_out as the page's 2-D [t, H * d] layout
    q2d = torch.full((t, H * d), 5.0, dtype=torch.bfloat16, device=DEV)
    run(x, s, q_out=q2d)
    assert mla.prolog_last_fused()
    assert torch.equal(q2d.view(t, H, d), ref_q)


def test_repeatable():
    s = W.prolog_shapes()["prolog_small"]
    x = W.make_prolog_inputs(s, device=DEV)
    a = [t.clone() for t in run(x, s)]
    b = run(x, s)
    assert all(torch.equal(u, v) for u, v in zip(a, b))


def test_head_dim_outside_the_fused_kernel():
    # head_dim 96 is not a multiple of 128 (the fused kernel's N chunks): the library GEMM + row kernel path
    s = W.PrologShape("prolog_d96", tokens=50, hidden=256, q_lora_rank=96, num_heads=3, head_dim=96, rope_dim=32,
                      seed=64)
    x = W.make_prolog_inputs(s, device=DEV)
    q, kv, cq = run(x, s)
    assert not mla.prolog_last_fused()
    check_all(x, s, np.arange(s.tokens), q, kv, cq)
