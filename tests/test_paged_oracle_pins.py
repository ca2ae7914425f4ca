"""Pins for the paged KV-cache gather oracle (oracle/paged.py).

Hand-worked cases (tests/golden/paged_cases.json), plus properties fixed by
the definition: an identity block table over a contiguous cache returns each
sequence's prefix; relabelling physical blocks does not change the result;
cumulative lengths equal plain lengths; a start offset s equals loading s more
tokens and dropping the first s.  Planted mistakes in copies of the oracle's
source must each fail one of these checks.
"""
import json
import os
import types

import numpy as np
import pytest

import oracle.paged as paged

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "paged_cases.json")


def _golden_caches(doc):
    nb, bs = doc["num_blocks"], doc["block_size"]
    k = np.array([[10 * b + s for s in range(bs)] for b in range(nb)], dtype=np.int32).reshape(nb, bs, 1, 1)
    return k, k + 100


def check_golden(mod):
    fails = []
    doc = json.load(open(GOLDEN))
    kc, vc = _golden_caches(doc)
    for c in doc["cases"]:
        key, value, bad = mod.paged_cache_load(kc, vc, np.array(c["block_tables"]), c["context_lens"],
                                               c["seq_starts"], c["cumsum"])
        if key.reshape(-1).tolist() != c["key"] or value.reshape(-1).tolist() != c["value"]:
            fails.append("%s: got %s / %s" % (c["name"], key.reshape(-1).tolist(), value.reshape(-1).tolist()))
        if sorted(bad) != c["bad"]:
            fails.append("%s: bad rows %s want %s" % (c["name"], bad, c["bad"]))
    return fails


def _random_problem(rng, batch=3, bs=4, H=2, D=3, W=5):
    nb = batch * W + 2
    kc = rng.integers(-1000, 1000, size=(nb, bs, H, D)).astype(np.int16)
    vc = rng.integers(-1000, 1000, size=(nb, bs, H, D + 1)).astype(np.int16)
    perm = rng.permutation(nb)[: batch * W].reshape(batch, W)
    lens = rng.integers(0, bs * W, size=batch)
    return kc, vc, perm, lens


def check_properties(mod):
    fails = []
    rng = np.random.default_rng(3)
    for trial in range(4):
        kc, vc, table, lens = _random_problem(rng)
        batch, W = table.shape
        bs = kc.shape[1]
        # identity table over a contiguous cache: each sequence's prefix, in order
        seqs = rng.integers(-50, 50, size=(batch, W * bs, 2, 3)).astype(np.int16)
        cont = seqs.reshape(batch * W, bs, 2, 3)
        ident = np.arange(batch * W).reshape(batch, W)
        key, _, bad = mod.paged_cache_load(cont, cont, ident, lens)
        want = np.concatenate([seqs[b, : lens[b]] for b in range(batch)]) if lens.sum() else key
        if bad or not np.array_equal(key, want):
            fails.append("identity table trial %d" % trial)
        # relabelling physical blocks (cache and table together) changes nothing
        key0, val0, _ = mod.paged_cache_load(kc, vc, table, lens)
        relabel = rng.permutation(kc.shape[0])
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[relabel], vc2[relabel] = kc, vc
        key1, val1, _ = mod.paged_cache_load(kc2, vc2, relabel[table], lens)
        if not (np.array_equal(key0, key1) and np.array_equal(val0, val1)):
            fails.append("relabel trial %d" % trial)
        # cumulative lengths == plain lengths
        c = np.concatenate([[7], 7 + np.cumsum(lens)])
        key2, val2, _ = mod.paged_cache_load(kc, vc, table, c, cumsum=True)
        if not (np.array_equal(key0, key2) and np.array_equal(val0, val2)):
            fails.append("cumsum trial %d" % trial)
        # start offsets: load [s, s + len) == load [0, s + len) and drop the first s rows
        starts = np.minimum(rng.integers(0, 5, size=batch), W * bs - lens)
        key3, _, _ = mod.paged_cache_load(kc, vc, table, lens, seq_starts=starts)
        key4, _, _ = mod.paged_cache_load(kc, vc, table, lens + starts)
        _, offs4, _ = mod.lengths_and_offsets(lens + starts, False)
        want = np.concatenate([key4[offs4[b] + starts[b]: offs4[b] + starts[b] + lens[b]] for b in range(batch)])
        if not np.array_equal(key3, want):
            fails.append("start offsets trial %d" % trial)
    return fails


CHECKS = [check_golden, check_properties]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_paged_oracle_pin(check):
    fails = check(paged)
    assert not fails, "\n".join(fails[:10])


MUTATIONS = {
    "slot_from_block_index": ("lb, within = pos // block_size, pos % block_size",
                              "lb, within = pos // block_size, (pos // block_size) % block_size"),
    "starts_ignored": ("pos = start + t", "pos = t"),
    "cumsum_off_by_one": ("lens = [c[b + 1] - c[b] for b in range(len(c) - 1)]",
                          "lens = [c[b + 1] - c[b] + 1 for b in range(len(c) - 1)]"),
    "table_transposed": ("blk = int(tables[b, lb]) if 0 <= lb < width else -1",
                         "blk = int(tables[lb % tables.shape[0], b % width]) if 0 <= lb < width else -1"),
    "bad_rows_not_flagged": ("                bad.append(row)\n", ""),
    "value_from_key_cache": ("value[row] = value_cache[blk, within]", "value[row] = key_cache[blk, within, :, :1]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_paged_pins_catch_planted_mistakes(name):
    src = open(paged.__file__).read()
    old, new = MUTATIONS[name]
    assert old in src, name
    mod = types.ModuleType("paged_bad")
    exec(compile(src.replace(old, new), "paged_bad", "exec"), mod.__dict__)
    caught = []
    for check in CHECKS:
        try:
            if check(mod):
                caught.append(check.__name__)
        except Exception as e:  # a crash also counts as caught
            caught.append("%s (%s)" % (check.__name__, type(e).__name__))
    assert caught, "planted mistake %s passed every pin" % name
