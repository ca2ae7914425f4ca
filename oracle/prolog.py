"""MLA Prolog oracle (non-quantised path) -- test infrastructure only.

Plain fp64 statement of the "MlaProlog" page (cann-recipes-infer, 功能说明 /
计算公式 / 参数说明 sections), which turns hidden states x into the query and the
key-value latent of MLA:

    c^Q = RmsNorm(x . wq_a)                      (weight gamma_cq)
    q   = RmsNorm(c^Q . wq_b)                    (weight 1: "the second RmsNorm's
                                                  weight is constantly 1")
    q[..., -rope_dim:]  = ROPE(q[..., -rope_dim:])   in place, interleaved
    kv  = RmsNorm(x . wkv)                       (weight gamma_ckv)
    kv[..., -rope_dim:] = ROPE(kv[..., -rope_dim:])  in place, interleaved

Readings where the page is silent (each one also listed in the design notes):
  * RmsNorm(v) = v / sqrt(mean(v^2) + eps) * gamma over the last axis; eps is
    not printed, so it is a parameter (default 1e-6).
  * q is normalised per head: c^Q . wq_b is viewed as [t, num_heads, head_dim]
    (the q_out shape), and the norm and the rope act on the -1 axis of that
    view -- the only reading under which "the last rope_dim channels" is one
    slice per head.
  * "Interleaved" rope rotates adjacent pairs (2i, 2i+1) of the rope slice:
        y[2i]   = x[2i]   * cos[2i]   - x[2i+1] * sin[2i]
        y[2i+1] = x[2i+1] * cos[2i+1] + x[2i]   * sin[2i+1]
    with rope_cos / rope_sin [t, rope_dim] indexed by token and channel.
  * c^Q enters the second projection as a bf16 tensor (round to nearest even):
    the page's quantised variant hands c^Q to wq_b as a low-precision tensor
    (qr_out), and every activation the page types is bf16.  ``round_cq=False``
    gives the unrounded chain.
  * The projections x . wq_a, c^Q . wq_b and x . wkv are exact (fp64 here).

Only tests/ and the benchmark's CPU baseline use this module; it shares no code
with the CUDA path.  The matrix products are numpy matmuls (a library primitive
standing for one step); every other step is written out below in the page's
order.
"""
import numpy as np


def f64(a):
    """fp64 copy of a numpy array or a CPU torch tensor (bf16 widened exactly)."""
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def round_bf16(v):
    """Round fp64 values to the nearest bf16 value (ties to even); finite normal range."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                   # v = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # 8 significant bits


def rms_norm(v, gamma, eps):
    """v / sqrt(mean(v^2) + eps) * gamma over the last axis."""
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * gamma


def rope_interleaved(v, cos, sin):
    """Rotates adjacent channel pairs (2i, 2i+1) of v by the given cos / sin (same shape as v)."""
    out = np.empty_like(v)
    even, odd = v[..., 0::2], v[..., 1::2]
    out[..., 0::2] = even * cos[..., 0::2] - odd * sin[..., 0::2]
    out[..., 1::2] = odd * cos[..., 1::2] + even * sin[..., 1::2]
    return out


def mla_prolog_q(c_q, wq_b, rope_cos, rope_sin, num_heads, eps=1e-6):
    """The query half after c^Q: q = RmsNorm(c^Q . wq_b) per head (weight 1), then the interleaved
    rope on each head's last rope_dim channels.  Returns q [t, num_heads, head_dim] in fp64."""
    c_q, wq_b = f64(c_q), f64(wq_b)
    cos, sin = f64(rope_cos), f64(rope_sin)
    t = c_q.shape[0]
    head_dim = wq_b.shape[1] // num_heads
    rope_dim = cos.shape[1]
    q = (c_q @ wq_b).reshape(t, num_heads, head_dim)
    q = rms_norm(q, 1.0, eps)
    q[..., head_dim - rope_dim:] = rope_interleaved(q[..., head_dim - rope_dim:], cos[:, None, :], sin[:, None, :])
    return q


def mla_prolog(token_x, wq_a, wq_b, wkv, rope_cos, rope_sin, gamma_cq, gamma_ckv, num_heads, eps=1e-6,
               round_cq=True):
    """Returns (q [t, num_heads, head_dim], kv [t, head_dim], c^Q [t, q_lora_rank]) in fp64.

    token_x [t, h], wq_a [h, q_lora_rank], wq_b [q_lora_rank, num_heads * head_dim],
    wkv [h, head_dim], rope_cos / rope_sin [t, rope_dim], gamma_cq [q_lora_rank],
    gamma_ckv [head_dim].
    """
    x = f64(token_x)
    wq_a, wq_b, wkv = f64(wq_a), f64(wq_b), f64(wkv)
    cos, sin = f64(rope_cos), f64(rope_sin)
    gamma_cq, gamma_ckv = f64(gamma_cq), f64(gamma_ckv)
    t = x.shape[0]
    head_dim = wkv.shape[1]
    rope_dim = cos.shape[1]
    assert wq_b.shape[1] == num_heads * head_dim and rope_dim % 2 == 0 and rope_dim <= head_dim

    # query: down-projection and first RmsNorm
    c_q = rms_norm(x @ wq_a, gamma_cq, eps)
    if round_cq:
        c_q = round_bf16(c_q)
    q = mla_prolog_q(c_q, wq_b, cos, sin, num_heads, eps)
    # key-value latent: down-projection, RmsNorm, interleaved rope on the last rope_dim channels
    kv = rms_norm(x @ wkv, gamma_ckv, eps)
    kv[..., head_dim - rope_dim:] = rope_interleaved(kv[..., head_dim - rope_dim:], cos, sin)
    return q, kv, c_q
