"""B200 (sm_100a) varlen causal MLA prefill.

Python binding of ``libmla_prefill.so`` (C ABI in ``include/mla_prefill.h``).
This module only marshals torch tensors into ``mla_tensor`` descriptors and
forwards them; every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
import ctypes
import os

from . import workloads  # noqa: F401  (seeded synthetic inputs)

__all__ = [
    "MLA_MASK_NONE", "MLA_MASK_CAUSAL", "MlaError", "load_library", "mla_prefill", "mla_prefill_noalloc",
    "mla_prefill_get_workspace_size", "mla_prefill_ws", "mla_prefill_ws_status",
    "mla_paged_cache_load", "mla_prefill_paged", "mla_prolog", "set_split_tiles", "set_kernel", "mla_prefill_device_status", "mla_status_string", "prefill",
    "workloads",
]

MLA_F16, MLA_BF16, MLA_I32, MLA_I8 = 0, 1, 2, 3
MLA_MASK_NONE, MLA_MASK_CAUSAL = 0, 1
STATUS_NAMES = {
    0: "MLA_OK", 1: "MLA_ERR_NULL", 2: "MLA_ERR_DTYPE", 3: "MLA_ERR_SHAPE", 4: "MLA_ERR_ALIGN",
    5: "MLA_ERR_HEADS", 6: "MLA_ERR_UNSUPPORTED", 7: "MLA_ERR_CUDA", 8: "MLA_ERR_SEQLEN",
    9: "MLA_ERR_DEVICE_TIMEOUT", 10: "MLA_ERR_INDEX", 11: "MLA_ERR_WORKSPACE",
}

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_prefill.so")


class MlaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class MlaError(RuntimeError):
    def __init__(self, code, where="mla_prefill"):
        self.code = int(code)
        super().__init__("%s failed: %s (%d)" % (where, mla_status_string(code), self.code))


_lib = None


def load_library(path=None):
    """Load (once) and return the ctypes handle of libmla_prefill.so."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError("libmla_prefill.so not built (run `python -m mla_prefill_attention_varlen_b200.build`)")
    lib = ctypes.CDLL(p)
    T = ctypes.POINTER(MlaTensor)
    lib.mla_prefill.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, T,
                                ctypes.c_void_p]
    lib.mla_prefill.restype = ctypes.c_int
    lib.mla_prefill_device_status.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
    lib.mla_prefill_device_status.restype = ctypes.c_int
    lib.mla_status_string.argtypes = [ctypes.c_int]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_prefill_noalloc.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_float, T, ctypes.c_void_p]
    lib.mla_prefill_noalloc.restype = ctypes.c_int
    lib.mla_prefill_get_workspace_size.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_float, T, ctypes.POINTER(ctypes.c_uint64)]
    lib.mla_prefill_get_workspace_size.restype = ctypes.c_int
    lib.mla_prefill_ws.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, T,
                                   ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p]
    lib.mla_prefill_ws.restype = ctypes.c_int
    lib.mla_prefill_ws_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
    lib.mla_prefill_ws_status.restype = ctypes.c_int
    lib.mla_paged_cache_load.argtypes = [T, T, T, T, T, ctypes.c_int, T, T, ctypes.c_void_p]
    lib.mla_paged_cache_load.restype = ctypes.c_int
    lib.mla_prefill_paged.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                      T, ctypes.c_void_p]
    lib.mla_prefill_paged.restype = ctypes.c_int
    lib.mla_prolog.argtypes = [T, T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_float, T, T, T, ctypes.c_void_p]
    lib.mla_prolog.restype = ctypes.c_int
    lib.mla_prefill_set_profile_events.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.mla_prefill_set_profile_events.restype = ctypes.c_int
    lib.mla_selftest_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_void_p]
    lib.mla_selftest_wait_timeout.restype = ctypes.c_int
    lib.mla_prefill_last_launches.argtypes = []
    lib.mla_prefill_last_launches.restype = ctypes.c_int
    lib.mla_prefill_last_kernel.argtypes = []
    lib.mla_prefill_last_kernel.restype = ctypes.c_int
    lib.mla_prolog_set_path.argtypes = [ctypes.c_int]
    lib.mla_prolog_set_path.restype = ctypes.c_int
    lib.mla_prolog_last_fused.argtypes = []
    lib.mla_prolog_last_fused.restype = ctypes.c_int
    lib.mla_prefill_set_kernel.argtypes = [ctypes.c_int]
    lib.mla_prefill_set_kernel.restype = ctypes.c_int
    lib.mla_prefill_set_split_tiles.argtypes = [ctypes.c_int]
    lib.mla_prefill_set_split_tiles.restype = ctypes.c_int
    lib.mla_prefill_version.argtypes = []
    lib.mla_prefill_version.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def mla_status_string(code):
    try:
        return load_library().mla_status_string(int(code)).decode()
    except ImportError:
        return STATUS_NAMES.get(int(code), "unknown")


def _dtype_code(t):
    import torch

    return {torch.float16: MLA_F16, torch.bfloat16: MLA_BF16, torch.int32: MLA_I32, torch.int8: MLA_I8}.get(t.dtype,
                                                                                                        -1)


def as_mla_tensor(t):
    """Describe a torch tensor (any device) as an mla_tensor; no copy."""
    d = MlaTensor()
    d.data = t.data_ptr() if t.numel() > 0 or t.data_ptr() else None
    d.dtype = _dtype_code(t)
    d.ndim = t.dim()
    if d.ndim > 4:
        raise ValueError("at most 4 dimensions")
    for i in range(d.ndim):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream_handle(stream, device):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def mla_prefill(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out,
                stream=None):
    """Call the C ABI ``mla_prefill`` on torch tensors (same argument order).

    All tensors must live on the current CUDA device; ``out`` is written in
    place.  ``stream``: a torch.cuda.Stream, a raw handle, or None for the
    current stream.  Raises MlaError on any non-zero status.
    """
    lib = load_library()
    descs = [as_mla_tensor(t) for t in (q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, out)]
    rc = lib.mla_prefill(*(ctypes.byref(d) for d in descs[:7]), int(mask_type), int(head_num), int(kv_head_num),
                         float(qk_scale), ctypes.byref(descs[7]), _stream_handle(stream, q.device))
    if rc != 0:
        raise MlaError(rc)
    return out


def mla_prefill_noalloc(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num,
                        qk_scale, out, stream=None):
    """Call the C ABI ``mla_prefill_noalloc``: same as ``mla_prefill`` but the
    library allocates no device memory (its scratch is a fixed static array;
    see include/mla_prefill.h for the size limit and the sharing rules)."""
    lib = load_library()
    descs = [as_mla_tensor(t) for t in (q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, out)]
    rc = lib.mla_prefill_noalloc(*(ctypes.byref(d) for d in descs[:7]), int(mask_type), int(head_num),
                                 int(kv_head_num), float(qk_scale), ctypes.byref(descs[7]),
                                 _stream_handle(stream, q.device))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_noalloc")
    return out


def mla_prefill_get_workspace_size(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num,
                                   qk_scale, out):
    """Call the C ABI ``mla_prefill_get_workspace_size``: bytes of device workspace ``mla_prefill_ws``
    needs for these arguments (only shapes, strides, dtypes and scalars are read)."""
    lib = load_library()
    descs = [as_mla_tensor(t) for t in (q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, out)]
    n = ctypes.c_uint64(0)
    rc = lib.mla_prefill_get_workspace_size(*(ctypes.byref(d) for d in descs[:7]), int(mask_type), int(head_num),
                                            int(kv_head_num), float(qk_scale), ctypes.byref(descs[7]),
                                            ctypes.byref(n))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_get_workspace_size")
    return n.value


def mla_prefill_ws(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out,
                   workspace, stream=None):
    """Call the C ABI ``mla_prefill_ws``: ``mla_prefill`` with a caller-owned workspace (a uint8 CUDA
    tensor, 256-byte aligned, at least ``mla_prefill_get_workspace_size`` bytes)."""
    lib = load_library()
    descs = [as_mla_tensor(t) for t in (q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, out)]
    rc = lib.mla_prefill_ws(*(ctypes.byref(d) for d in descs[:7]), int(mask_type), int(head_num), int(kv_head_num),
                            float(qk_scale), ctypes.byref(descs[7]), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream_handle(stream, q.device))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_ws")
    return out


def mla_prefill_ws_status(workspace, stream=None):
    """Synchronise the stream and return the status of the last ``mla_prefill_ws`` call on ``workspace``."""
    lib = load_library()
    st = ctypes.c_int(0)
    rc = lib.mla_prefill_ws_status(workspace.data_ptr(), _stream_handle(stream, workspace.device), ctypes.byref(st))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_ws_status")
    return st.value


def prefill(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, head_num, kv_head_num, qk_scale,
            mask_type=MLA_MASK_CAUSAL, out=None, stream=None):
    """Allocate ``out`` [T_q, H, 128] (if not given) and run ``mla_prefill``."""
    import torch

    if out is None:
        out = torch.empty(q.shape[0], head_num, v.shape[-1] if v.dim() == 3 else 128, dtype=q.dtype,
                          device=q.device)
    return mla_prefill(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale,
                       out, stream)


def mla_paged_cache_load(key_cache, value_cache, block_tables, context_lens, key, value, seq_starts=None,
                         cumsum=False, stream=None):
    """Call the C ABI ``mla_paged_cache_load`` (gather a paged K/V cache into packed key / value)."""
    lib = load_library()
    d = [as_mla_tensor(t) for t in (key_cache, value_cache, block_tables, context_lens, key, value)]
    ss = ctypes.byref(as_mla_tensor(seq_starts)) if seq_starts is not None else None
    rc = lib.mla_paged_cache_load(ctypes.byref(d[0]), ctypes.byref(d[1]), ctypes.byref(d[2]), ctypes.byref(d[3]),
                                  ss, 1 if cumsum else 0, ctypes.byref(d[4]), ctypes.byref(d[5]),
                                  _stream_handle(stream, key.device))
    if rc != 0:
        raise MlaError(rc, "mla_paged_cache_load")
    return key, value


def mla_prefill_paged(q, q_rope, key_cache, value_cache, block_tables, q_seqlen, kv_seqlen, mask_type, head_num,
                      kv_head_num, qk_scale, out, stream=None):
    """Call the C ABI ``mla_prefill_paged``: prefill attention reading K / K_rope / V in place from
    paged caches (key_cache [blocks, block_size, G, 192] = K_nope | K_rope, value_cache
    [blocks, block_size, G, 128]) through block_tables [batch, W]."""
    lib = load_library()
    d = [as_mla_tensor(t) for t in (q, q_rope, key_cache, value_cache, block_tables, q_seqlen, kv_seqlen, out)]
    rc = lib.mla_prefill_paged(*(ctypes.byref(x) for x in d[:7]), int(mask_type), int(head_num), int(kv_head_num),
                               float(qk_scale), ctypes.byref(d[7]), _stream_handle(stream, q.device))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_paged")
    return out


def mla_prolog(token_x, wq_a, wq_b, wkv, rope_cos, rope_sin, gamma_cq, gamma_ckv, num_heads, q_out, kv_out,
               cq_out=None, eps=1e-6, stream=None):
    """Call the C ABI ``mla_prolog`` (MLA Prolog, non-quantised): writes q_out [t, H, d],
    kv_out [t, d] and, if given, cq_out [t, q_lora_rank] (bf16) in place."""
    lib = load_library()
    d = [as_mla_tensor(t) for t in (token_x, wq_a, wq_b, wkv, rope_cos, rope_sin, gamma_cq, gamma_ckv, q_out,
                                    kv_out)]
    cq = ctypes.byref(as_mla_tensor(cq_out)) if cq_out is not None else None
    rc = lib.mla_prolog(*(ctypes.byref(x) for x in d[:8]), int(num_heads), float(eps), ctypes.byref(d[8]),
                        ctypes.byref(d[9]), cq, _stream_handle(stream, token_x.device))
    if rc != 0:
        raise MlaError(rc, "mla_prolog")
    return q_out, kv_out


def set_split_tiles(tiles):
    """Split-KV chunk (in 128-key tiles) for later prefill calls on this thread: -1 automatic, 0 off."""
    rc = load_library().mla_prefill_set_split_tiles(int(tiles))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_set_split_tiles")


def set_kernel(kernel):
    """Attention kernel for later prefill calls on this thread: -1 automatic, 1 single-CTA, 2 CTA pair."""
    rc = load_library().mla_prefill_set_kernel(int(kernel))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_set_kernel")


def set_prolog_path(path):
    """q projection of later mla_prolog calls on this thread: -1 the fused tcgen05 kernel where the
    sizes allow it (default), 0 the library GEMM + row kernel."""
    rc = load_library().mla_prolog_set_path(int(path))
    if rc != 0:
        raise MlaError(rc, "mla_prolog_set_path")


def prolog_last_fused():
    """True if the last mla_prolog call of this thread ran the fused q kernel."""
    return bool(load_library().mla_prolog_last_fused())


def set_profile_events(start=None, stop=None):
    """Record torch.cuda.Events around the attention-kernel launch of later calls."""
    lib = load_library()
    if start is None or stop is None:
        lib.mla_prefill_set_profile_events(None, None)
        return
    for ev in (start, stop):
        if not ev.cuda_event:  # torch creates the CUDA event on its first record
            ev.record()
    if not (start.cuda_event and stop.cuda_event):
        raise RuntimeError("could not create CUDA events")
    lib.mla_prefill_set_profile_events(start.cuda_event, stop.cuda_event)


def mla_prefill_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device status word."""
    import torch

    lib = load_library()
    st = ctypes.c_int(0)
    rc = lib.mla_prefill_device_status(_stream_handle(stream, torch.cuda.current_device()), ctypes.byref(st))
    if rc != 0:
        raise MlaError(rc, "mla_prefill_device_status")
    return st.value
