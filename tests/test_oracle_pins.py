"""Pins for the fp64 CPU oracle: checks against things other than itself.

Each check ties the oracle to something the "MLA Prefill" page or plain
mathematics fixes:

* hand-worked examples (``tests/golden/hand_cases.json``, each derived by hand
  from the page's members table);
* a library attention routine (torch ``scaled_dot_product_attention`` in fp64,
  with an explicit bottom-right causal mask) on the special case where the
  rope part is concatenated onto the nope part;
* closed forms: qkScale = 0 gives the mean of the visible V rows, a single
  visible key gives that key's V row exactly, rows with no visible key give 0,
  a huge qkScale gives the V row of the best-scoring key;
* invariants: weights sum to 1 and masked weights are exactly 0;
* identities: nope + rope split equals one concatenated product, a sequence in
  a batch equals the same sequence alone, row sampling equals the full run.

``test_pins_catch_planted_mistakes`` compiles deliberately broken copies of
the oracle's C source on the CPU and shows that these checks reject each one.
"""
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from oracle import MASK_CAUSAL, MASK_NONE

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "hand_cases.json")
TOL = 1e-12


def _problem(rng, lens_q, lens_k, H, G, dn=5, r=3, dv=4, extra_tokens=0):
    tq, tk = sum(lens_q) + extra_tokens, sum(lens_k)
    return dict(
        q=rng.standard_normal((tq, H, dn)), q_rope=rng.standard_normal((tq, H, r)),
        k=rng.standard_normal((tk, G, dn)), k_rope=rng.standard_normal((tk, G, r)),
        v=rng.standard_normal((tk, G, dv)),
        q_seqlen=np.array(lens_q, dtype=np.int32), kv_seqlen=np.array(lens_k, dtype=np.int32),
        head_num=H, kv_head_num=G)


def _run(orc, p, qk_scale, mask_type=MASK_CAUSAL, rows=None):
    return orc.prefill(p["q"], p["q_rope"], p["k"], p["k_rope"], p["v"], p["q_seqlen"], p["kv_seqlen"],
                       p["head_num"], p["kv_head_num"], qk_scale, mask_type=mask_type, rows=rows)


def _visible_count(i, lq, lk, causal):
    """How many keys query row i sees: min(Lk, i + Lk - Lq + 1) clipped at 0, or Lk."""
    if not causal:
        return lk
    return int(min(lk, max(0, i + lk - lq + 1)))


# ---------------------------------------------------------------------------
# checks, each returning a list of failure messages (empty = pass)
# ---------------------------------------------------------------------------

def check_hand_cases(orc):
    fails = []
    doc = json.load(open(GOLDEN))
    for c in doc["cases"]:
        arr = {k: np.array(c[k], dtype=np.float64) for k in ("q", "q_rope", "k", "k_rope", "v")}
        out = orc.prefill(arr["q"], arr["q_rope"], arr["k"], arr["k_rope"], arr["v"], c["q_seqlen"],
                          c["kv_seqlen"], c["head_num"], c["kv_head_num"], c["qk_scale"], mask_type=c["mask_type"])
        for t, exp in enumerate(c["expected"]):
            if exp is None:
                if not np.all(np.isnan(out[t])):
                    fails.append("%s: token %d should be untouched" % (c["name"], t))
            elif not np.allclose(out[t], np.array(exp), rtol=0, atol=TOL):
                fails.append("%s: token %d got %s want %s" % (c["name"], t, out[t].tolist(), exp))
        if "probs" in c:
            pr = c["probs"]
            p, _ = orc.row_probs(arr["q"], arr["q_rope"], arr["k"], arr["k_rope"], c["q_seqlen"], c["kv_seqlen"],
                                 c["head_num"], c["kv_head_num"], c["qk_scale"], pr["token"], pr["head"],
                                 mask_type=c["mask_type"])
            if not np.allclose(p, pr["p"], rtol=0, atol=TOL):
                fails.append("%s: probs %s want %s" % (c["name"], p.tolist(), pr["p"]))
    return fails


def _sdpa_reference(p, qk_scale, causal):
    """torch SDPA (fp64, CPU) per sequence on [Qn||Qr] . [Kn||Kr]^T with an explicit mask."""
    H, G = p["head_num"], p["kv_head_num"]
    g = H // G
    q = torch.from_numpy(np.concatenate([p["q"], p["q_rope"]], axis=2))
    k = torch.from_numpy(np.concatenate([p["k"], p["k_rope"]], axis=2))
    v = torch.from_numpy(p["v"])
    out = np.full((q.shape[0], H, v.shape[2]), np.nan)
    has_key = np.zeros((q.shape[0],), dtype=bool)
    cq = ck = 0
    scale = float(np.float32(qk_scale))
    for lq, lk in zip(p["q_seqlen"].tolist(), p["kv_seqlen"].tolist()):
        if lq > 0 and lk > 0:
            qs = q[cq:cq + lq].permute(1, 0, 2)[None]  # [1, H, Lq, D]
            ks = k[ck:ck + lk].permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
            vs = v[ck:ck + lk].permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
            i = torch.arange(lq)[:, None]
            j = torch.arange(lk)[None, :]
            mask = (j <= i + (lk - lq)) if causal else torch.ones(lq, lk, dtype=torch.bool)
            o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask, scale=scale)
            out[cq:cq + lq] = o[0].permute(1, 0, 2).numpy()
            has_key[cq:cq + lq] = mask.any(dim=1).numpy()
        cq += lq
        ck += lk
    return out, has_key


SDPA_SHAPES = [
    # (lens_q, lens_k, H, G, r)
    ([5], [5], 1, 1, 3),
    ([3, 17], [3, 17], 4, 2, 3),
    ([2, 5], [5, 9], 2, 2, 3),       # chunked: Lq < Lk, bottom-right
    ([5, 1], [3, 1], 4, 1, 3),       # Lq > Lk: leading rows see nothing
    ([1, 2, 3], [1, 2, 3], 4, 4, 0),  # no rope part at all
    ([17], [17], 2, 1, 3),
]


def check_sdpa(orc):
    fails = []
    rng = np.random.default_rng(11)
    for n, (lq, lk, H, G, r) in enumerate(SDPA_SHAPES):
        p = _problem(rng, lq, lk, H, G, r=r)
        for mask_type in (MASK_CAUSAL, MASK_NONE):
            scale = 0.37
            got = _run(orc, p, scale, mask_type)
            ref, has_key = _sdpa_reference(p, scale, mask_type == MASK_CAUSAL)
            err = np.abs(got[has_key] - ref[has_key]).max() if has_key.any() else 0.0
            if not err <= 1e-12:
                fails.append("sdpa shape %d mask %d: max err %g" % (n, mask_type, err))
            if not np.all(got[~has_key] == 0.0):
                fails.append("sdpa shape %d mask %d: rows with no key are not 0" % (n, mask_type))
    return fails


def check_closed_forms(orc):
    fails = []
    rng = np.random.default_rng(12)
    for lq, lk in ([7], [7]), ([3, 6], [8, 6]), ([6], [4]):
        p = _problem(rng, lq, lk, 4, 2)
        # qkScale = 0: every visible score is equal -> O_i is the mean of the visible V rows.
        got = _run(orc, p, 0.0)
        cq = ck = 0
        for a, b in zip(lq, lk):
            for i in range(a):
                n = _visible_count(i, a, b, True)
                for h in range(4):
                    want = p["v"][ck:ck + n, h // 2].mean(axis=0) if n else np.zeros(p["v"].shape[2])
                    if not np.allclose(got[cq + i, h], want, rtol=0, atol=TOL):
                        fails.append("mean closed form lq=%s row %d head %d" % (lq, i, h))
            cq += a
            ck += b
    # one visible key -> exactly that key's V row (p = 1 exactly)
    p = _problem(rng, [4, 3], [4, 3], 2, 2)
    got = _run(orc, p, 0.9)
    for t, kt in ((0, 0), (4, 4)):
        if not np.array_equal(got[t], p["v"][kt]):
            fails.append("single visible key: token %d" % t)
    # huge scale: the softmax becomes the argmax of the visible scores
    p = _problem(rng, [6], [6], 2, 1)
    got = _run(orc, p, 1e4)
    for i in range(6):
        for h in range(2):
            s = p["q"][i, h] @ p["k"][: i + 1, 0].T + p["q_rope"][i, h] @ p["k_rope"][: i + 1, 0].T
            want = p["v"][int(np.argmax(s)), 0]
            if not np.allclose(got[i, h], want, rtol=0, atol=1e-9):
                fails.append("argmax limit row %d head %d" % (i, h))
    return fails


def check_invariants(orc):
    fails = []
    rng = np.random.default_rng(13)
    lq, lk = [3, 9, 4], [5, 9, 2]
    p = _problem(rng, lq, lk, 4, 2)
    cq = 0
    for a, b in zip(lq, lk):
        for i in range(a):
            for h in range(4):
                for mask_type in (MASK_CAUSAL, MASK_NONE):
                    w, n = orc.row_probs(p["q"], p["q_rope"], p["k"], p["k_rope"], p["q_seqlen"], p["kv_seqlen"],
                                         4, 2, 0.5, cq + i, h, mask_type=mask_type)
                    nv = _visible_count(i, a, b, mask_type == MASK_CAUSAL)
                    if n != nv:
                        fails.append("visible count row %d: %d want %d" % (i, n, nv))
                    if np.any(w[nv:] != 0.0):
                        fails.append("masked weight not exactly 0 (row %d)" % i)
                    if nv and abs(w.sum() - 1.0) > 1e-14:
                        fails.append("weights do not sum to 1 (row %d): %r" % (i, w.sum()))
                    if np.any(w[:nv] <= 0.0):
                        fails.append("visible weight not positive (row %d)" % i)
        cq += a
    return fails


def check_identities(orc):
    fails = []
    rng = np.random.default_rng(14)
    p = _problem(rng, [6, 11, 1], [9, 11, 3], 4, 2)
    base = _run(orc, p, 0.41)
    # nope + rope split == one product over the concatenated dims
    cat = dict(p)
    cat["q"] = np.concatenate([p["q"], p["q_rope"]], axis=2)
    cat["k"] = np.concatenate([p["k"], p["k_rope"]], axis=2)
    cat["q_rope"] = np.zeros(p["q_rope"].shape[:2] + (0,))
    cat["k_rope"] = np.zeros(p["k_rope"].shape[:2] + (0,))
    if not np.allclose(_run(orc, cat, 0.41), base, rtol=0, atol=TOL):
        fails.append("split identity")
    # each sequence alone == the same sequence inside the batch (bit-identical)
    cq = ck = 0
    for lq, lk in zip(p["q_seqlen"].tolist(), p["kv_seqlen"].tolist()):
        one = dict(p, q=p["q"][cq:cq + lq], q_rope=p["q_rope"][cq:cq + lq], k=p["k"][ck:ck + lk],
                   k_rope=p["k_rope"][ck:ck + lk], v=p["v"][ck:ck + lk],
                   q_seqlen=np.array([lq], np.int32), kv_seqlen=np.array([lk], np.int32))
        if not np.array_equal(_run(orc, one, 0.41), base[cq:cq + lq]):
            fails.append("batch invariance (seq at %d)" % cq)
        cq += lq
        ck += lk
    # a row subset equals the full run on those rows and leaves the others untouched
    rows = [0, 5, 7, 16]
    sub = _run(orc, p, 0.41, rows=rows)
    if not np.array_equal(sub[rows], base[rows]):
        fails.append("row sampling")
    others = np.setdiff1d(np.arange(base.shape[0]), rows)
    if not np.all(np.isnan(sub[others])):
        fails.append("row sampling touched other rows")
    # GQA: H = 2G equals H = G with each kv head repeated per query head
    rep = dict(p, k=np.repeat(p["k"], 2, axis=1), k_rope=np.repeat(p["k_rope"], 2, axis=1),
               v=np.repeat(p["v"], 2, axis=1), kv_head_num=4)
    if not np.array_equal(_run(orc, rep, 0.41), base):
        fails.append("GQA == repeated KV")
    return fails


ALL_CHECKS = [check_hand_cases, check_sdpa, check_closed_forms, check_invariants, check_identities]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    fails = check(oracle)
    assert not fails, "\n".join(fails[:20])


@settings(max_examples=80, deadline=None, derandomize=True)
@given(st.data())
def test_oracle_matches_library_attention_on_random_shapes(data):
    # the library pin over drawn ragged shapes: empty sequences, Lq > Lk and Lq < Lk, GQA ratios,
    # no rope part, both masks, negative and zero scales
    batch = data.draw(st.integers(1, 4))
    lens_q = data.draw(st.lists(st.integers(0, 12), min_size=batch, max_size=batch))
    lens_k = data.draw(st.lists(st.integers(0, 12), min_size=batch, max_size=batch))
    G = data.draw(st.sampled_from([1, 2, 3]))
    H = G * data.draw(st.sampled_from([1, 2, 3]))
    r = data.draw(st.sampled_from([0, 2, 3]))
    scale = data.draw(st.floats(-2.0, 2.0, allow_nan=False))
    mask_type = data.draw(st.sampled_from([MASK_CAUSAL, MASK_NONE]))
    p = _problem(np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1))), lens_q, lens_k, H, G, r=r)
    got = _run(oracle, p, scale, mask_type)
    ref, has_key = _sdpa_reference(p, scale, mask_type == MASK_CAUSAL)
    if has_key.any():
        assert np.abs(got[has_key] - ref[has_key]).max() <= TOL
    assert np.all(got[~has_key] == 0.0)


def test_oracle_rejects_inconsistent_seqlens():
    rng = np.random.default_rng(15)
    p = _problem(rng, [3], [3], 1, 1)
    with pytest.raises(ValueError):
        oracle.prefill(p["q"], p["q_rope"], p["k"], p["k_rope"], p["v"], [4], [3], 1, 1, 1.0)
    with pytest.raises(ValueError):
        oracle.prefill(p["q"], p["q_rope"], p["k"], p["k_rope"], p["v"], [-1], [3], 1, 1, 1.0)
    with pytest.raises(ValueError):
        oracle.prefill(p["q"], p["q_rope"], p["k"], p["k_rope"], p["v"], [3], [3], 1, 1, 1.0, mask_type=7)


def test_qk_scale_is_a_float32():
    # qkScale is a float argument: 1/sqrt(192) reaches the oracle as its float32 rounding.
    rng = np.random.default_rng(16)
    p = _problem(rng, [4], [4], 1, 1)
    exact = 1.0 / math.sqrt(192.0)
    f32 = float(np.float32(exact))
    assert f32 != exact
    w1, _ = oracle.row_probs(p["q"], p["q_rope"], p["k"], p["k_rope"], [4], [4], 1, 1, exact, 3, 0)
    s = (p["q"][3, 0] @ p["k"][:, 0].T + p["q_rope"][3, 0] @ p["k_rope"][:, 0].T) * f32
    want = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
    assert np.allclose(w1, want, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# planted mistakes: each broken copy of the oracle must fail some pin
# ---------------------------------------------------------------------------

MUTATIONS = {
    "rope_term_dropped": ("dot += qr[r] * kr[r];", "dot += 0.0 * qr[r] * kr[r];"),
    "mask_top_left": ("const int64_t off = lk - lq;", "const int64_t off = 0;"),
    "head_map_modulo": ("const int64_t kh = h / group;", "const int64_t kh = h % pb->kv_head_num;"),
    "softmax_sign": ("p[j] = exp(p[j] - m);", "p[j] = exp(m - p[j]);"),
    "scale_ignored": ("p[j] = pb->scale * dot;", "p[j] = dot;"),
    "no_renormalise": ("if (vis) p[j] /= denom;", "if (vis) p[j] /= 1.0;"),
    "v_packing_offset_dropped": ("const double *vr = pb->v + ((pb->ck[b] + j)", "const double *vr = pb->v + ((j)"),
    "k_transposed_layout": ("const double *kn = pb->k + ((pb->ck[b] + j) * pb->kv_head_num + kh) * pb->d_nope;",
                            "const double *kn = pb->k + (kh * pb->t_k + (pb->ck[b] + j)) * pb->d_nope;"),
    "mask_strict": ("(j <= i + off) : 1;\n        if (!vis)", "(j < i + off) : 1;\n        if (!vis)"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mla_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert old in src, "mutation anchor missing: %s" % name
    bad_src = tmp_path / "mla_oracle_bad.c"
    bad_src.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_bad.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(lib), str(bad_src), "-lm"],
                   check=True)
    bad = oracle.Oracle(str(lib))
    caught = []
    for check in ALL_CHECKS:
        try:
            if check(bad):
                caught.append(check.__name__)
        except Exception as e:  # a crash or rejection also counts as caught
            caught.append("%s (%s)" % (check.__name__, type(e).__name__))
    assert caught, "planted mistake %s passed every pin" % name
