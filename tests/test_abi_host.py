"""C ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest
import torch

import mla_prefill_attention_varlen_b200 as mla
from mla_prefill_attention_varlen_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mla.load_library()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(HEADER_DIR, fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ \*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n.startswith("mla_")))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("mla_prefill", "mla_prefill_device_status", "mla_status_string", "mla_prefill_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), "missing export %s" % n


def test_library_is_built_for_sm100a_only():
    # the nvcc command line names exactly one target, sm_100a (no PTX for other architectures)
    flags = build.NVCC_FLAGS
    targets = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert targets == ["arch=compute_100a,code=sm_100a"]
    assert not any(f.startswith(("-arch", "--gpu-architecture", "--generate-code")) for f in flags)


def test_status_strings(lib):
    for code, name in mla.STATUS_NAMES.items():
        assert lib.mla_status_string(code).decode().startswith(name)
    assert lib.mla_status_string(12345).decode() == "unknown mla_status"
    assert lib.mla_prefill_version() >= 100


# ---------------------------------------------------------------------------
# Host-side validation.  These descriptors point at host memory that is never
# dereferenced: every call below must be rejected before any CUDA call.
# ---------------------------------------------------------------------------

def make_args(T=256, Tk=256, H=4, G=2, batch=2, dtype=torch.bfloat16):
    t = dict(
        q=torch.zeros(T, H, 128, dtype=dtype), q_rope=torch.zeros(T, H, 64, dtype=dtype),
        k=torch.zeros(Tk, G, 128, dtype=dtype), k_rope=torch.zeros(Tk, G, 64, dtype=dtype),
        v=torch.zeros(Tk, G, 128, dtype=dtype), q_seqlen=torch.zeros(batch, dtype=torch.int32),
        kv_seqlen=torch.zeros(batch, dtype=torch.int32), out=torch.zeros(T, H, 128, dtype=dtype))
    return t, H, G


def call(lib, t, H, G, mask=1, scale=0.5, override=None):
    d = {k: mla.as_mla_tensor(v) for k, v in t.items()}
    for k, fn in (override or {}).items():
        fn(d[k])
    p = lambda k: ctypes.byref(d[k]) if d[k] is not None else None
    return lib.mla_prefill(p("q"), p("q_rope"), p("k"), p("k_rope"), p("v"), p("q_seqlen"), p("kv_seqlen"), mask, H,
                           G, scale, p("out"), None)


def test_rejects_null(lib):
    t, H, G = make_args()
    d = {k: mla.as_mla_tensor(v) for k, v in t.items()}
    rc = lib.mla_prefill(None, ctypes.byref(d["q_rope"]), ctypes.byref(d["k"]), ctypes.byref(d["k_rope"]),
                         ctypes.byref(d["v"]), ctypes.byref(d["q_seqlen"]), ctypes.byref(d["kv_seqlen"]), 1, H, G,
                         0.5, ctypes.byref(d["out"]), None)
    assert rc == 1

    def null_data(x):
        x.data = None
    assert call(lib, t, H, G, override={"v": null_data}) == 1


@pytest.mark.parametrize("H,G", [(0, 1), (4, 0), (4, 3), (-1, 1)])
def test_rejects_bad_heads(lib, H, G):
    t, _, _ = make_args()
    assert call(lib, t, H, G) == 5


def test_rejects_heads_not_matching_shapes(lib):
    t, H, G = make_args()
    assert call(lib, t, 8, G) == 3  # q is [T, 4, 128]
    assert call(lib, t, H, 4) == 3  # k is [T, 2, 128]


def test_rejects_dtypes(lib):
    t, H, G = make_args()
    t["v"] = t["v"].half()
    assert call(lib, t, H, G) == 2
    t, H, G = make_args()
    t["q_seqlen"] = t["q_seqlen"].long()
    assert call(lib, t, H, G) == 2
    t, H, G = make_args(dtype=torch.float32)
    assert call(lib, t, H, G) == 2


def test_rejects_shapes(lib):
    t, H, G = make_args()
    t["q_rope"] = torch.zeros(255, H, 64, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 3
    t, H, G = make_args()
    t["k"] = torch.zeros(256, G, 96, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 3
    t, H, G = make_args()
    t["kv_seqlen"] = torch.zeros(3, dtype=torch.int32)
    assert call(lib, t, H, G) == 3
    t, H, G = make_args()
    t["out"] = torch.zeros(256, H, 64, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 3


def test_padded_kv_layout_checks(lib):
    # the page's padded [batch, max_seq, kv_head*embeddimV] form: all of K, K_rope, V or none
    t, H, G = make_args(batch=2)
    t["k"] = torch.zeros(2, 128, G * 128, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 6  # K padded, K_rope / V packed
    t["k_rope"] = torch.zeros(2, 128, G * 64, dtype=torch.bfloat16)
    t["v"] = torch.zeros(2, 128, G * 128, dtype=torch.bfloat16)
    if not torch.cuda.is_available():
        assert call(lib, t, H, G) == 7  # valid: passes host validation, then needs CUDA
    t["v"] = torch.zeros(2, 100, G * 128, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 3  # max_seq differs between K and V
    wide = torch.zeros(2, 256, G * 128, dtype=torch.bfloat16)
    t["v"] = wide[:, :128]  # batch rows not dense
    assert call(lib, t, H, G) == 6
    t, H, G = make_args(batch=3)
    t["k"] = torch.zeros(2, 128, G * 128, dtype=torch.bfloat16)
    t["k_rope"] = torch.zeros(2, 128, G * 64, dtype=torch.bfloat16)
    t["v"] = torch.zeros(2, 128, G * 128, dtype=torch.bfloat16)
    assert call(lib, t, H, G) == 3  # padded batch differs from len(q_seqlen)


def test_rejects_misalignment(lib):
    t, H, G = make_args()

    def shift(x):
        x.data = x.data + 2
    assert call(lib, t, H, G, override={"q": shift}) == 4

    def odd_stride(x):
        x.stride[0] = 4 * 128 + 4
    assert call(lib, t, H, G, override={"k": odd_stride}) == 4

    def inner_stride(x):
        x.stride[2] = 2
    assert call(lib, t, H, G, override={"v": inner_stride}) == 4


def test_rejects_mask_scale_and_alias(lib):
    t, H, G = make_args()
    assert call(lib, t, H, G, mask=2) == 6
    assert call(lib, t, H, G, scale=float("inf")) == 6
    assert call(lib, t, H, G, scale=float("nan")) == 6
    t, H, G = make_args(H=2, G=2)
    t["out"] = t["v"]  # out aliasing an input
    assert call(lib, t, H, G) == 6


def test_accepts_2d_and_strided_views_on_host(lib):
    # a well-formed call passes validation and only then reaches CUDA; with no
    # GPU the result is MLA_ERR_CUDA (7), with a GPU the data would be device memory.
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    t, H, G = make_args()
    t["q"] = t["q"].reshape(256, H * 128)
    wide = torch.zeros(256, H, 192, dtype=torch.bfloat16)
    t["q_rope"] = wide[:, :, 128:]
    assert call(lib, t, H, G) == 7


def test_empty_batch_is_a_no_op(lib):
    t, H, G = make_args(batch=0)
    assert call(lib, t, H, G) == 0


# ---------------------------------------------------------------------------
# caller-owned workspace: the size query and the host-side checks of mla_prefill_ws
# ---------------------------------------------------------------------------

def _align(x, a=256):
    return (x + a - 1) // a * a


def expected_workspace_bytes(batch, t_q, t_k, split=0, heads=0, key_extent=None):
    """The workspace mla_prefill_ws needs, section by section (each rounded up to 256 bytes): the
    status header, a 16-byte counter block, per-sequence offsets {cq, ck, Lq, Lk} (16 bytes each),
    per-sequence unit offsets (batch + 1 ints), the key-tile histogram (ceil(T_k/128) + 2 ints) and
    the unit list (ceil(T_q/256) + batch int pairs); with split-KV chunks of `split` key tiles also
    the per-unit entry offsets, the entry table and the fp32 partial rows (O / l and the
    log-sum-exp) of every entry, head and row of a 256-row unit."""
    units = -(-t_q // 256) + batch
    n = 256 + _align(16) + _align(16 * batch) + _align(4 * (batch + 1)) + _align(4 * (-(-t_k // 128) + 2)) \
        + _align(8 * units)
    if split:
        tiles = -(-(key_extent or t_k) // 128)
        # the chunk doubles while the fp32 partial rows (129 floats per row) would pass 2 GiB
        while split < tiles and units * max(1, -(-tiles // split)) * heads * 256 * 129 * 4 > 2 << 30:
            split *= 2
        if split >= tiles:
            return n
        entries = units * max(1, -(-tiles // split))
        n += _align(4 * (units + 1)) + _align(8 * entries) + _align(4 * entries * heads * 256) \
            + _align(4 * entries * heads * 256 * 128)
    return n


def ws_size(lib, t, H, G, mask=1, scale=0.5):
    d = {k: mla.as_mla_tensor(v) for k, v in t.items()}
    n = ctypes.c_uint64(0)
    rc = lib.mla_prefill_get_workspace_size(*(ctypes.byref(d[k]) for k in ("q", "q_rope", "k", "k_rope", "v",
                                                                            "q_seqlen", "kv_seqlen")),
                                            mask, H, G, scale, ctypes.byref(d["out"]), ctypes.byref(n))
    return rc, n.value


@pytest.mark.parametrize("T,Tk,batch,H,G", [(256, 256, 2, 4, 2), (1000, 5000, 7, 8, 8), (1, 1, 1, 1, 1),
                                            (40000, 70000, 300, 2, 1)])
def test_workspace_size_formula(lib, T, Tk, batch, H, G):
    # explicit split settings: the size needs no GPU (only the automatic mode reads the SM count)
    t, _, _ = make_args(T=T, Tk=Tk, H=H, G=G, batch=batch)
    try:
        mla.set_split_tiles(0)
        rc, n = ws_size(lib, t, H, G)
        assert rc == 0 and n == expected_workspace_bytes(batch, T, Tk)
        mla.set_split_tiles(3)
        rc, n = ws_size(lib, t, H, G)
        tiles = -(-Tk // 128)
        expect = expected_workspace_bytes(batch, T, Tk, split=3 if 3 < tiles else 0, heads=H)
        assert rc == 0 and n == expect
    finally:
        mla.set_split_tiles(-1)


def test_workspace_size_and_call_reject_bad_arguments(lib):
    t, H, G = make_args()
    d = {k: mla.as_mla_tensor(v) for k, v in t.items()}
    args = [ctypes.byref(d[k]) for k in ("q", "q_rope", "k", "k_rope", "v", "q_seqlen", "kv_seqlen")]
    assert lib.mla_prefill_get_workspace_size(*args, 1, H, G, 0.5, ctypes.byref(d["out"]), None) == 1
    assert ws_size(lib, t, 8, G)[0] == 3  # argument errors as in mla_prefill
    try:
        mla.set_split_tiles(0)
        rc, need = ws_size(lib, t, H, G)
        assert rc == 0
        buf = torch.zeros(need + 512, dtype=torch.uint8)
        base = (buf.data_ptr() + 255) // 256 * 256  # never dereferenced: rejected on the host
        assert lib.mla_prefill_ws(*args, 1, H, G, 0.5, ctypes.byref(d["out"]), None, need, None) == 1
        assert lib.mla_prefill_ws(*args, 1, H, G, 0.5, ctypes.byref(d["out"]), base, need - 1, None) == 11
        assert lib.mla_prefill_ws(*args, 1, H, G, 0.5, ctypes.byref(d["out"]), base + 16, need, None) == 11
        assert lib.mla_prefill_ws(*args, 1, 8, G, 0.5, ctypes.byref(d["out"]), base, need, None) == 3
    finally:
        mla.set_split_tiles(-1)
    st = ctypes.c_int(0)
    assert lib.mla_prefill_ws_status(None, None, ctypes.byref(st)) == 1
    assert lib.mla_prefill_ws_status(buf.data_ptr() | 8, None, ctypes.byref(st)) == 11


# ---------------------------------------------------------------------------
# mla_paged_cache_load host-side validation (descriptors are never dereferenced)
# ---------------------------------------------------------------------------

def paged_args(nb=6, bs=16, H=2, Dk=64, Dv=64, batch=2, W=4, T=40, dtype=torch.bfloat16):
    return dict(kc=torch.zeros(nb, bs, H, Dk, dtype=dtype), vc=torch.zeros(nb, bs, H, Dv, dtype=dtype),
                table=torch.zeros(batch, W, dtype=torch.int32), lens=torch.zeros(batch, dtype=torch.int32),
                key=torch.zeros(T, H, Dk, dtype=dtype), value=torch.zeros(T, H, Dv, dtype=dtype))


def paged_call(lib, a, starts=None, cumsum=0):
    d = {k: mla.as_mla_tensor(v) for k, v in a.items()}
    s = ctypes.byref(mla.as_mla_tensor(starts)) if starts is not None else None
    return lib.mla_paged_cache_load(ctypes.byref(d["kc"]), ctypes.byref(d["vc"]), ctypes.byref(d["table"]),
                                    ctypes.byref(d["lens"]), s, cumsum, ctypes.byref(d["key"]),
                                    ctypes.byref(d["value"]), None)


def test_paged_rejects_bad_arguments(lib):
    a = paged_args()
    if not torch.cuda.is_available():
        assert paged_call(lib, a) == 7  # well formed: reaches CUDA
    b = dict(a, key=torch.zeros(40, 2, 64, dtype=torch.float16))
    assert paged_call(lib, b) == 2  # output dtype differs from its cache
    b = dict(a, lens=torch.zeros(3, dtype=torch.int32))
    assert paged_call(lib, b) == 3  # plain lengths must be [batch]
    assert paged_call(lib, dict(a, lens=torch.zeros(3, dtype=torch.int32)), cumsum=1) in (0, 7)  # [batch+1] ok
    b = dict(a, kc=torch.zeros(6, 16, 1, 64, dtype=torch.bfloat16), key=torch.zeros(40, 1, 64, dtype=torch.bfloat16))
    assert paged_call(lib, b) == 3  # value cache heads differ from key cache heads
    b = dict(a, kc=torch.zeros(6, 16, 2, 3, dtype=torch.bfloat16), key=torch.zeros(40, 2, 3, dtype=torch.bfloat16))
    assert paged_call(lib, b) == 4  # 12-byte rows are not whole 16-byte vectors
    b = dict(a, table=torch.zeros(2, 4, dtype=torch.int64))
    assert paged_call(lib, b) == 2
    assert paged_call(lib, a, starts=torch.zeros(3, dtype=torch.int32)) == 3
    b = dict(a, value=a["key"])
    assert paged_call(lib, b) == 6  # outputs overlap


# ---------------------------------------------------------------------------
# mla_prefill_paged host-side validation (descriptors are never dereferenced)
# ---------------------------------------------------------------------------

def prefill_paged_args(T=64, H=4, G=2, nb=8, bs=16, W=4, batch=2, dtype=torch.bfloat16):
    return dict(q=torch.zeros(T, H, 128, dtype=dtype), q_rope=torch.zeros(T, H, 64, dtype=dtype),
                kc=torch.zeros(nb, bs, G, 192, dtype=dtype), vc=torch.zeros(nb, bs, G, 128, dtype=dtype),
                table=torch.zeros(batch, W, dtype=torch.int32), q_seqlen=torch.zeros(batch, dtype=torch.int32),
                kv_seqlen=torch.zeros(batch, dtype=torch.int32), out=torch.zeros(T, H, 128, dtype=dtype)), H, G


def prefill_paged_call(lib, a, H, G, mask=1, scale=0.5):
    d = {k: mla.as_mla_tensor(v) for k, v in a.items()}
    r = lambda k: ctypes.byref(d[k])
    return lib.mla_prefill_paged(r("q"), r("q_rope"), r("kc"), r("vc"), r("table"), r("q_seqlen"), r("kv_seqlen"),
                                 mask, H, G, scale, r("out"), None)


@pytest.mark.parametrize("bs,ok", [(8, True), (16, True), (64, True), (128, True), (256, True), (384, True),
                                   (4, False), (12, False), (48, False), (96, False), (136, False), (200, False)])
def test_prefill_paged_block_sizes(lib, bs, ok):
    a, H, G = prefill_paged_args(bs=bs)
    rc = prefill_paged_call(lib, a, H, G)
    if ok:
        if not torch.cuda.is_available():
            assert rc == 7  # well formed: reaches CUDA
    else:
        assert rc == 6


def test_prefill_paged_rejects_bad_arguments(lib):
    a, H, G = prefill_paged_args()
    d = {k: mla.as_mla_tensor(v) for k, v in a.items()}
    assert lib.mla_prefill_paged(ctypes.byref(d["q"]), ctypes.byref(d["q_rope"]), None, ctypes.byref(d["vc"]),
                                 ctypes.byref(d["table"]), ctypes.byref(d["q_seqlen"]), ctypes.byref(d["kv_seqlen"]),
                                 1, H, G, 0.5, ctypes.byref(d["out"]), None) == 1
    b = dict(a, kc=torch.zeros(8, 16, G, 128, dtype=torch.bfloat16))
    assert prefill_paged_call(lib, b, H, G) == 3  # key cache must be 192 wide (nope | rope)
    b = dict(a, vc=torch.zeros(9, 16, G, 128, dtype=torch.bfloat16))
    assert prefill_paged_call(lib, b, H, G) == 3  # block counts differ
    b = dict(a, vc=torch.zeros(8, 32, G, 128, dtype=torch.bfloat16))
    assert prefill_paged_call(lib, b, H, G) == 3  # block sizes differ
    b = dict(a, kc=torch.zeros(8, 16, 1, 192, dtype=torch.bfloat16))
    assert prefill_paged_call(lib, b, H, G) == 3  # kv heads differ from kv_head_num
    b = dict(a, vc=torch.zeros(8, 16, G, 128, dtype=torch.float16))
    assert prefill_paged_call(lib, b, H, G) == 2  # cache dtype differs from q
    b = dict(a, table=torch.zeros(2, 4, dtype=torch.int64))
    assert prefill_paged_call(lib, b, H, G) == 2
    b = dict(a, table=torch.zeros(3, 4, dtype=torch.int32))
    assert prefill_paged_call(lib, b, H, G) == 3  # table rows != batch
    b = dict(a, table=torch.zeros(4, 2, dtype=torch.int32).t())
    assert prefill_paged_call(lib, b, H, G) == 4  # table rows not contiguous
    wide = torch.zeros(8, 16, G, 200, dtype=torch.bfloat16)
    b = dict(a, kc=wide[..., 4:196])
    assert prefill_paged_call(lib, b, H, G) == 4  # 8-byte base offset
    wide = torch.zeros(8, 16, G, 196, dtype=torch.bfloat16)
    b = dict(a, kc=wide[..., :192])
    assert prefill_paged_call(lib, b, H, G) == 4  # head stride not a multiple of 8 elements
    assert prefill_paged_call(lib, a, 4, 3) == 5
    assert prefill_paged_call(lib, a, H, G, mask=5) == 6
    buf = torch.zeros(8 * 16 * G * 192 + 64 * H * 128, dtype=torch.bfloat16)
    b = dict(a, kc=buf[:8 * 16 * G * 192].view(8, 16, G, 192), out=buf[8 * 16 * G * 192 - 128:][:64 * H * 128]
             .view(64, H, 128))
    assert prefill_paged_call(lib, b, H, G) == 6  # out overlaps the key cache


def test_prefill_paged_empty_batch_is_a_no_op(lib):
    a, H, G = prefill_paged_args(batch=0)
    assert prefill_paged_call(lib, a, H, G) == 0


# ---------------------------------------------------------------------------
# mla_prolog host-side validation (descriptors are never dereferenced)
# ---------------------------------------------------------------------------

def prolog_args(t=8, h=64, r=32, H=2, d=32, R=16, dtype=torch.bfloat16):
    z = lambda *s: torch.zeros(*s, dtype=dtype)
    return dict(x=z(t, h), wq_a=z(h, r), wq_b=z(r, H * d), wkv=z(h, d), cos=z(t, R), sin=z(t, R), g_cq=z(r),
                g_ckv=z(d), q=z(t, H, d), kv=z(t, d), cq=z(t, r)), H


def prolog_call(lib, a, H, eps=1e-6, with_cq=True):
    d = {k: mla.as_mla_tensor(v) for k, v in a.items()}
    r = lambda k: ctypes.byref(d[k])
    return lib.mla_prolog(r("x"), r("wq_a"), r("wq_b"), r("wkv"), r("cos"), r("sin"), r("g_cq"), r("g_ckv"), H, eps,
                          r("q"), r("kv"), r("cq") if with_cq else None, None)


def test_prolog_accepts_well_formed_arguments(lib):
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    a, H = prolog_args()
    assert prolog_call(lib, a, H) == 7  # reaches CUDA
    assert prolog_call(lib, a, H, with_cq=False) == 7
    a["q"] = a["q"].reshape(8, H * 32)  # [t, H*d] form
    assert prolog_call(lib, a, H) == 7
    a, H = prolog_args(t=0)
    assert prolog_call(lib, a, H) == 0  # no tokens: nothing to do


def test_prolog_rejects_bad_arguments(lib):
    a, H = prolog_args()
    assert prolog_call(lib, a, 0) == 5
    assert prolog_call(lib, a, H, eps=-1.0) == 6
    assert prolog_call(lib, a, H, eps=float("nan")) == 6
    assert prolog_call(lib, dict(a, wkv=a["wkv"].half()), H) == 2
    assert prolog_call(lib, dict(a, g_cq=torch.zeros(32, dtype=torch.float32)), H) == 2
    assert prolog_call(lib, dict(a, wq_a=torch.zeros(48, 32, dtype=torch.bfloat16)), H) == 3  # h mismatch
    assert prolog_call(lib, dict(a, wq_b=torch.zeros(32, 48, dtype=torch.bfloat16)), H) == 3  # not H*d wide
    assert prolog_call(lib, dict(a, sin=torch.zeros(8, 8, dtype=torch.bfloat16)), H) == 3  # cos / sin widths
    assert prolog_call(lib, dict(a, cos=torch.zeros(7, 16, dtype=torch.bfloat16)), H) == 3  # one row per token
    assert prolog_call(lib, dict(a, kv=torch.zeros(8, 16, dtype=torch.bfloat16)), H) == 3
    assert prolog_call(lib, dict(a, q=torch.zeros(8, 3, 32, dtype=torch.bfloat16)), H) == 3
    assert prolog_call(lib, dict(a, g_ckv=torch.zeros(16, dtype=torch.bfloat16)), H) == 3
    a2, _ = prolog_args(R=6, d=32)
    assert prolog_call(lib, a2, H) == 4  # a 6-wide cos row stride is not a multiple of 8 elements
    a3, _ = prolog_args(R=40, d=32)
    assert prolog_call(lib, a3, H) == 6  # rope wider than the head
    wide = torch.zeros(8, 72, dtype=torch.bfloat16)
    assert prolog_call(lib, dict(a, x=wide[:, 4:68]), H) == 4  # 8-byte offset base
    assert prolog_call(lib, dict(a, x=torch.zeros(8, 68, dtype=torch.bfloat16)[:, :64]), H) == 4  # row stride 68
    buf = torch.zeros(8 * 64 + 8 * 32, dtype=torch.bfloat16)
    assert prolog_call(lib, dict(a, kv=buf[:256].view(8, 32), cq=buf[128:384].view(8, 32)), H) == 6  # outputs overlap
    assert prolog_call(lib, dict(a, kv=a["x"][:, :32]), H) == 6  # output over an input


def test_split_tiles_control(lib):
    assert lib.mla_prefill_set_split_tiles(-1) == 0
    assert lib.mla_prefill_set_split_tiles(0) == 0
    assert lib.mla_prefill_set_split_tiles(7) == 0
    assert lib.mla_prefill_set_split_tiles(-2) == 6
    assert lib.mla_prefill_set_split_tiles(-1) == 0


def test_last_launches_is_zero_without_work(lib):
    t, H, G = make_args(batch=0)
    assert call(lib, t, H, G) == 0
    assert lib.mla_prefill_last_launches() == 0
