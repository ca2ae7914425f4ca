"""Pins for the MLA Prolog oracle (oracle/prolog.py), none of them the oracle against itself.

* Hand-worked cases (tests/golden/prolog_cases.json, each with its derivation):
  per-head normalisation, interleaved pairs, each token's own cos / sin, eps
  inside the square root, zero input.
* Library special cases: torch's fp64 ``rms_norm`` for the norms, and the
  rope as multiplication by a unit complex number exp(i theta) on the pairs
  viewed as complex values (cos / sin equal within each pair).
* Invariances fixed by the formulas: scaling one head's wq_b columns or the
  whole input (eps = 0) changes nothing; tokens are independent; the rope
  keeps each pair's length and composes by adding angles; only the last
  rope_dim channels of each head are rotated.
* The bf16 rounding helper against torch's float32 -> bfloat16 conversion.
Planted mistakes in copies of the oracle's source must each fail one of these checks.
"""
import json
import os
import types

import numpy as np
import pytest
import torch

import oracle.prolog as prolog

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "prolog_cases.json")


def check_golden(mod):
    fails = []
    for c in json.load(open(GOLDEN))["cases"]:
        a = {k: np.array(c[k], dtype=np.float64) for k in ("token_x", "wq_a", "wq_b", "wkv", "rope_cos", "rope_sin",
                                                         "gamma_cq", "gamma_ckv")}
        q, kv, cq = mod.mla_prolog(a["token_x"], a["wq_a"], a["wq_b"], a["wkv"], a["rope_cos"], a["rope_sin"],
                                   a["gamma_cq"], a["gamma_ckv"], c["num_heads"], eps=c["eps"], round_cq=False)
        for name, got in (("q", q), ("kv", kv), ("c_q", cq)):
            want = np.array(c[name], dtype=np.float64)
            if got.shape != want.shape or not np.allclose(got, want, rtol=0, atol=1e-12):
                fails.append("%s: %s = %s, want %s" % (c["name"], name, got.tolist(), want.tolist()))
    return fails


def _problem(rng, t=5, h=24, r=16, heads=3, d=12, rope=6, angles=None):
    x = rng.standard_normal((t, h))
    wq_a = rng.standard_normal((h, r)) / np.sqrt(h)
    wq_b = rng.standard_normal((r, heads * d)) / np.sqrt(r)
    wkv = rng.standard_normal((h, d)) / np.sqrt(h)
    if angles is None:
        angles = rng.uniform(-np.pi, np.pi, size=(t, rope // 2))
    cos = np.repeat(np.cos(angles), 2, axis=1)
    sin = np.repeat(np.sin(angles), 2, axis=1)
    g_cq = 1 + 0.3 * rng.standard_normal(r)
    g_ckv = 1 + 0.3 * rng.standard_normal(d)
    return dict(token_x=x, wq_a=wq_a, wq_b=wq_b, wkv=wkv, rope_cos=cos, rope_sin=sin, gamma_cq=g_cq,
                gamma_ckv=g_ckv), heads, angles


def _run(mod, a, heads, eps=1e-6, round_cq=False):
    return mod.mla_prolog(a["token_x"], a["wq_a"], a["wq_b"], a["wkv"], a["rope_cos"], a["rope_sin"], a["gamma_cq"],
                          a["gamma_ckv"], heads, eps=eps, round_cq=round_cq)


def _torch_reference(a, heads, eps):
    """Independent formulation: torch fp64 rms_norm, rope as a complex rotation of the pairs."""
    T = {k: torch.from_numpy(np.array(v, dtype=np.float64)) for k, v in a.items()}
    x = T["token_x"]
    r, d, rope = T["wq_a"].shape[1], T["wkv"].shape[1], T["rope_cos"].shape[1]
    cq = torch.nn.functional.rms_norm(x @ T["wq_a"], (r,), weight=T["gamma_cq"], eps=eps)
    q = torch.nn.functional.rms_norm((cq @ T["wq_b"]).view(x.shape[0], heads, d), (d,), eps=eps)
    kv = torch.nn.functional.rms_norm(x @ T["wkv"], (d,), weight=T["gamma_ckv"], eps=eps)
    rot = torch.polar(torch.ones_like(T["rope_cos"][:, 0::2]), torch.atan2(T["rope_sin"][:, 0::2],
                                                                          T["rope_cos"][:, 0::2]))

    def rope_c(v, rot):
        z = torch.view_as_complex(v[..., d - rope:].contiguous().view(*v.shape[:-1], rope // 2, 2))
        out = v.clone()
        out[..., d - rope:] = torch.view_as_real(z * rot).reshape(*v.shape[:-1], rope)
        return out
    return rope_c(q, rot[:, None, :]).numpy(), rope_c(kv, rot).numpy(), cq.numpy()


def check_library(mod):
    fails = []
    rng = np.random.default_rng(11)
    for trial, eps in enumerate((1e-6, 0.0, 0.5)):
        a, heads, _ = _problem(rng)
        got = _run(mod, a, heads, eps)
        want = _torch_reference(a, heads, eps)
        for name, g, w in zip(("q", "kv", "c_q"), got, want):
            if g.shape != w.shape or np.abs(g - w).max() > 1e-12:
                fails.append("library trial %d: %s differs" % (trial, name))
    return fails


def check_invariances(mod):
    fails = []
    rng = np.random.default_rng(12)
    a, heads, angles = _problem(rng)
    q, kv, cq = _run(mod, a, heads, eps=0.0)
    d = a["wkv"].shape[1]
    rope = a["rope_cos"].shape[1]
    # scaling one head's up-projection columns leaves q unchanged (per-head norm)
    b = dict(a, wq_b=a["wq_b"].copy())
    b["wq_b"][:, d:2 * d] *= 7.5
    if np.abs(_run(mod, b, heads, eps=0.0)[0] - q).max() > 1e-12:
        fails.append("per-head scale changed q")
    # scaling the input leaves everything unchanged (eps = 0)
    s = _run(mod, dict(a, token_x=3.25 * a["token_x"]), heads, eps=0.0)
    if any(np.abs(u - v).max() > 1e-12 for u, v in zip(s, (q, kv, cq))):
        fails.append("input scale changed the result")
    # tokens are independent: a permutation of tokens (with their cos / sin) permutes the outputs
    perm = rng.permutation(a["token_x"].shape[0])
    pa = dict(a, token_x=a["token_x"][perm], rope_cos=a["rope_cos"][perm], rope_sin=a["rope_sin"][perm])
    pq, pkv, pcq = _run(mod, pa, heads, eps=0.0)
    if np.abs(pq - q[perm]).max() > 1e-12 or np.abs(pkv - kv[perm]).max() > 1e-12:
        fails.append("token permutation")
    # with angle 0 the rope is the identity: only the last rope_dim channels of each head move
    za = dict(a, rope_cos=np.ones_like(a["rope_cos"]), rope_sin=np.zeros_like(a["rope_sin"]))
    zq, zkv, _ = _run(mod, za, heads, eps=0.0)
    if np.abs(zq[..., :d - rope] - q[..., :d - rope]).max() > 1e-12 or \
            np.abs(zkv[..., :d - rope] - kv[..., :d - rope]).max() > 1e-12:
        fails.append("rope touched channels before the last rope_dim")
    # the rope keeps each pair's length ...
    pn = lambda v: np.hypot(v[..., d - rope::2], v[..., d - rope + 1::2])
    if np.abs(pn(q) - pn(zq)).max() > 1e-12 or np.abs(pn(kv) - pn(zkv)).max() > 1e-12:
        fails.append("rope changed a pair's length")
    # ... and two rotations compose by adding angles (rotate the rotated kv again through wkv = identity)
    h = a["token_x"].shape[1]
    ident = np.zeros((h, d))
    ident[:d, :d] = np.eye(d) if h >= d else ident[:d, :d]
    phi = rng.uniform(-np.pi, np.pi, size=angles.shape)
    cos2, sin2 = np.repeat(np.cos(phi), 2, axis=1), np.repeat(np.sin(phi), 2, axis=1)
    xin = np.zeros((a["token_x"].shape[0], h))
    xin[:, :d] = zkv
    one = dict(a, token_x=xin, wkv=ident, gamma_ckv=np.ones(d), rope_cos=a["rope_cos"], rope_sin=a["rope_sin"])
    _, kv1, _ = _run(mod, one, heads, eps=0.0)
    xin2 = np.zeros_like(xin)
    xin2[:, :d] = kv1
    _, kv2, _ = _run(mod, dict(one, token_x=xin2, rope_cos=cos2, rope_sin=sin2), heads, eps=0.0)
    tot = dict(one, rope_cos=np.repeat(np.cos(angles + phi), 2, axis=1),
               rope_sin=np.repeat(np.sin(angles + phi), 2, axis=1))
    _, kv12, _ = _run(mod, tot, heads, eps=0.0)
    if np.abs(kv2 - kv12).max() > 1e-12:
        fails.append("rotations do not compose")
    return fails


def check_round_bf16(mod):
    fails = []
    rng = np.random.default_rng(13)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    if not np.array_equal(mod.round_bf16(v.astype(np.float64)), want):
        fails.append("round_bf16 differs from torch float32 -> bfloat16")
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0])
    if mod.round_bf16(ties).tolist() != [1.0, 1 + 2 ** -6, -1.0, 0.0]:
        fails.append("round_bf16 ties: %s" % mod.round_bf16(ties).tolist())
    # c^Q really is rounded to bf16 on the default path
    a, heads, _ = _problem(rng)
    _, _, cq = _run(mod, a, heads, round_cq=True)
    if not np.array_equal(cq, mod.round_bf16(cq)) or np.array_equal(cq, _run(mod, a, heads)[2]):
        fails.append("c^Q is not rounded to bf16 when round_cq is set")
    return fails


CHECKS = [check_golden, check_library, check_invariances, check_round_bf16]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_prolog_oracle_pin(check):
    fails = check(prolog)
    assert not fails, "\n".join(fails[:10])


MUTATIONS = {
    "rope_half_split": ("even, odd = v[..., 0::2], v[..., 1::2]",
                        "even, odd = v[..., : v.shape[-1] // 2], v[..., v.shape[-1] // 2:]"),
    "rope_sign": ("out[..., 0::2] = even * cos[..., 0::2] - odd * sin[..., 0::2]",
                  "out[..., 0::2] = even * cos[..., 0::2] + odd * sin[..., 0::2]"),
    "rope_on_first_channels": ("q[..., head_dim - rope_dim:] = rope_interleaved(q[..., head_dim - rope_dim:]",
                               "q[..., :rope_dim] = rope_interleaved(q[..., :rope_dim]"),
    "norm_over_all_heads": ("    q = (c_q @ wq_b).reshape(t, num_heads, head_dim)\n    q = rms_norm(q, 1.0, eps)",
                            "    q = rms_norm(c_q @ wq_b, 1.0, eps).reshape(t, num_heads, head_dim)"),
    "gamma_cq_dropped": ("c_q = rms_norm(x @ wq_a, gamma_cq, eps)", "c_q = rms_norm(x @ wq_a, 1.0, eps)"),
    "sum_not_mean": ("ms = np.mean(v * v, axis=-1, keepdims=True)", "ms = np.sum(v * v, axis=-1, keepdims=True)"),
    "eps_outside_root": ("return v / np.sqrt(ms + eps) * gamma", "return v / (np.sqrt(ms) + eps) * gamma"),
    "first_token_angles": ("cos, sin = f64(rope_cos), f64(rope_sin)",
                           "cos, sin = f64(rope_cos)[:1].repeat(len(rope_cos), 0), f64(rope_sin)[:1].repeat(len(rope_sin), 0)"),
    "kv_without_rope": ("    kv[..., head_dim - rope_dim:] = rope_interleaved(kv[..., head_dim - rope_dim:], cos, sin)\n", ""),
    "round_truncates": ("np.rint(np.ldexp(m, 8))", "np.trunc(np.ldexp(m, 8))"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_prolog_pins_catch_planted_mistakes(name):
    src = open(prolog.__file__).read()
    old, new = MUTATIONS[name]
    assert old in src, name
    mod = types.ModuleType("prolog_bad")
    exec(compile(src.replace(old, new), "prolog_bad", "exec"), mod.__dict__)
    caught = []
    for check in CHECKS:
        try:
            if check(mod):
                caught.append(check.__name__)
        except Exception as e:  # a crash also counts as caught
            caught.append("%s (%s)" % (check.__name__, type(e).__name__))
    assert caught, "planted mistake %s passed every pin" % name
