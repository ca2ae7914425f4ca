"""fp64 CPU oracle for varlen causal MLA prefill -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may import this package.  It shares no code with
the CUDA path (``mla_prefill_attention_varlen_b200``) and never imports it.

The arithmetic lives in ``mla_oracle.c`` (plain C, fp64, one thread per core);
this module only marshals numpy arrays.  It follows the "MLA Prefill" page of
the Ascend Transformer Boost C API (the AtbMLAPreFillGetWorkspaceSize members
table: Q / QRope / K / kRope / V / qSeqLen / kvSeqLen / headNum / qkScale /
kvHeadNum / maskType / attenOut rows).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, a library attention routine on special cases, hand-worked examples and
invariants, not against itself.
"""
import ctypes
import os

import numpy as np

from . import build as _build

MASK_NONE = 0
MASK_CAUSAL = 1


def _bind(path):
    lib = ctypes.CDLL(path)
    d = ctypes.POINTER(ctypes.c_double)
    i32 = ctypes.POINTER(ctypes.c_int32)
    i64 = ctypes.POINTER(ctypes.c_int64)
    I = ctypes.c_int64
    lib.mla_oracle_prefill.argtypes = [d, d, d, d, d, i32, i32, I, I, I, I, I, I, I, I,
                                       ctypes.c_int, ctypes.c_float, i64, I, d, ctypes.c_int]
    lib.mla_oracle_prefill.restype = ctypes.c_int
    lib.mla_oracle_row_probs.argtypes = [d, d, d, d, i32, i32, I, I, I, I, I, I, I,
                                         ctypes.c_int, ctypes.c_float, I, I, d]
    lib.mla_oracle_row_probs.restype = ctypes.c_int64
    return lib


def _f64(a, ndim):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if a.ndim != ndim:
        raise ValueError("expected a %d-d array, got shape %s" % (ndim, a.shape))
    return a


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _as_np(x):
    """torch tensors (any float dtype) -> numpy; numpy passes through."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.is_floating_point():
            x = x.double()
        return x.numpy()
    return np.asarray(x)


class Oracle:
    """The oracle's entry points bound to one compiled copy of ``mla_oracle.c``.

    The default instance uses ``oracle/liboracle.so``; tests bind deliberately
    broken copies to show that the pins catch plausible mistakes.
    """

    def __init__(self, lib_path=None):
        self._path = lib_path
        self._lib = None

    def _load(self):
        if self._lib is None:
            self._lib = _bind(self._path or _build.build())
        return self._lib

    def prefill(self, q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, head_num, kv_head_num, qk_scale,
                mask_type=MASK_CAUSAL, rows=None, threads=0):
        return _prefill(self._load(), q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, head_num, kv_head_num,
                        qk_scale, mask_type, rows, threads)

    def row_probs(self, q, q_rope, k, k_rope, q_seqlen, kv_seqlen, head_num, kv_head_num, qk_scale, token,
                  head, mask_type=MASK_CAUSAL):
        return _row_probs(self._load(), q, q_rope, k, k_rope, q_seqlen, kv_seqlen, head_num, kv_head_num,
                          qk_scale, token, head, mask_type)


def _prefill(lib, q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, head_num, kv_head_num, qk_scale,
             mask_type, rows, threads):
    """attenOut for packed varlen MLA prefill, in fp64.

    q [T_q, H, Dn], q_rope [T_q, H, R], k [T_k, G, Dn], k_rope [T_k, G, R],
    v [T_k, G, Dv] (numpy or torch, any float dtype: values are widened to
    fp64 exactly); q_seqlen / kv_seqlen [batch] int.  ``qk_scale`` is rounded
    to float32 first, as the page's qkScale is a float.  ``rows``: optional
    packed token indices; only those rows are computed.  Returns out
    [T_q, H, Dv] float64 with NaN in every row that was not computed (rows
    not sampled, and tokens past sum(q_seqlen)).
    """
    q, q_rope, k, k_rope, v = (_f64(_as_np(x), 3) for x in (q, q_rope, k, k_rope, v))
    qs = np.ascontiguousarray(_as_np(q_seqlen), dtype=np.int32).reshape(-1)
    ks = np.ascontiguousarray(_as_np(kv_seqlen), dtype=np.int32).reshape(-1)
    if qs.shape != ks.shape:
        raise ValueError("q_seqlen and kv_seqlen must have the same length")
    t_q, h, dn = q.shape
    t_k, g, _ = k.shape
    r = q_rope.shape[2]
    dv = v.shape[2]
    if q_rope.shape[:2] != (t_q, h) or k_rope.shape != (t_k, g, r) or k.shape[2] != dn or v.shape[:2] != (t_k, g):
        raise ValueError("inconsistent shapes")
    if h != head_num or g != kv_head_num:
        raise ValueError("head counts do not match tensor shapes")
    out = np.full((t_q, h, dv), np.nan)
    if rows is not None:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        rows_p, n_rows = _ptr(rows_a, ctypes.c_int64), rows_a.size
    else:
        rows_p, n_rows = None, 0
    if r == 0:  # keep valid (unused) pointers for an empty rope part
        q_rope = np.zeros((t_q, h, 1))
        k_rope = np.zeros((t_k, g, 1))
    rc = lib.mla_oracle_prefill(
        _ptr(q, ctypes.c_double), _ptr(q_rope, ctypes.c_double), _ptr(k, ctypes.c_double),
        _ptr(k_rope, ctypes.c_double), _ptr(v, ctypes.c_double), _ptr(qs, ctypes.c_int32),
        _ptr(ks, ctypes.c_int32), qs.size, t_q, t_k, h, g, dn, r, dv, int(mask_type),
        float(qk_scale), rows_p, n_rows, _ptr(out, ctypes.c_double), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected the problem (code %d)" % rc)
    return out


def _row_probs(lib, q, q_rope, k, k_rope, q_seqlen, kv_seqlen, head_num, kv_head_num, qk_scale, token, head,
               mask_type):
    """Attention weights p[j], j < kv_seqlen[b], of one query row (packed token, head)."""
    q, q_rope, k, k_rope = (_f64(_as_np(x), 3) for x in (q, q_rope, k, k_rope))
    qs = np.ascontiguousarray(_as_np(q_seqlen), dtype=np.int32).reshape(-1)
    ks = np.ascontiguousarray(_as_np(kv_seqlen), dtype=np.int32).reshape(-1)
    t_q, h, dn = q.shape
    t_k, g, _ = k.shape
    r = q_rope.shape[2]
    if r == 0:
        q_rope = np.zeros((t_q, h, 1))
        k_rope = np.zeros((t_k, g, 1))
    p = np.zeros(max(int(ks.max()) if ks.size else 0, 1))
    n = lib.mla_oracle_row_probs(
        _ptr(q, ctypes.c_double), _ptr(q_rope, ctypes.c_double), _ptr(k, ctypes.c_double),
        _ptr(k_rope, ctypes.c_double), _ptr(qs, ctypes.c_int32), _ptr(ks, ctypes.c_int32), qs.size, t_q, t_k,
        h, g, dn, r, int(mask_type), float(qk_scale), int(token), int(head), _ptr(p, ctypes.c_double))
    if n < 0:
        raise ValueError("bad row")
    cq = np.concatenate([[0], np.cumsum(qs)])
    b = int(np.searchsorted(cq, token, side="right") - 1)
    return p[: int(ks[b])], int(n)


_default = Oracle()


def prefill(*args, **kwargs):
    """attenOut in fp64; see ``_prefill`` for the arguments."""
    return _default.prefill(*args, **kwargs)


def row_probs(*args, **kwargs):
    """Attention weights of one query row; see ``_row_probs``."""
    return _default.row_probs(*args, **kwargs)


def core_count():
    return os.cpu_count() or 1
