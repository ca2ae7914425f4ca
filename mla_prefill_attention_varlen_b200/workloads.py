"""Seeded synthetic workloads for varlen MLA prefill.

This module only draws inputs: shapes, sequence lengths and random values.  It
holds none of the attention arithmetic, so both the CUDA path's tests and the
CPU oracle can take their inputs from it without sharing any of the method.

Shapes follow the packed layouts of the "MLA Prefill" page (Q [nTokens, qhead,
embeddimV], QRope [nTokens, qhead, 64], K / V [batch*seq, kv_head, embeddimV],
kRope [batch*seq, kv_head, 64], qSeqLen / kvSeqLen [batch] int32).  Values are
i.i.d. normal, drawn in fp32 and rounded to the 16-bit dtype (round to nearest
even), so every consumer reads identical 16-bit values.
"""
import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

EMBED_DIM_V = 128  # embeddimV: nope width of Q/K and width of V
ROPE_DIM = 64      # QRope / kRope width


@dataclass
class Workload:
    name: str
    q_seqlens: List[int]
    kv_seqlens: List[int]
    head_num: int
    kv_head_num: int
    dtype: torch.dtype = torch.bfloat16
    std: float = 1.0
    seed: int = 0
    causal: bool = True
    d_nope: int = EMBED_DIM_V
    d_rope: int = ROPE_DIM
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.q_seqlens)

    @property
    def t_q(self) -> int:
        return int(sum(self.q_seqlens))

    @property
    def t_k(self) -> int:
        return int(sum(self.kv_seqlens))

    @property
    def qk_scale(self) -> float:
        """1/sqrt(192) rounded to float32 (qkScale is a float argument)."""
        return float(np.float32(1.0 / math.sqrt(self.d_nope + self.d_rope)))


def _config3_lengths() -> List[int]:
    # 16 lengths drawn uniformly from [128, 4096] (inclusive), fixed seed 0.
    return [int(x) for x in np.random.default_rng(0).integers(128, 4097, size=16)]


def workloads() -> dict:
    l3 = _config3_lengths()
    w = [
        Workload("tiny", [37, 64], [37, 64], 4, 4, seed=1,
                 description="batch=2, qSeqLen=kvSeqLen={37,64}, H=G=4, bf16 N(0,1), causal"),
        Workload("uniform", [1024] * 4, [1024] * 4, 16, 16, seed=2,
                 description="batch=4, L=1024, H=G=16, bf16 N(0,1), causal"),
        Workload("varlen_gqa", l3, l3, 32, 8, seed=3,
                 description="batch=16, L~U[128,4096] (numpy default_rng(0)), H=32, G=8, bf16 N(0,1), causal"),
        Workload("long", [16384], [16384], 128, 128, seed=4,
                 description="batch=1, L=16384, H=G=128, bf16 N(0,1), causal"),
        Workload("chunked", [512] * 8, [4096] * 8, 128, 128, dtype=torch.float16, std=0.5, seed=5,
                 description="batch=8, Lq=512, Lk=4096 (bottom-right causal), H=G=128, fp16 N(0,0.5)"),
    ]
    return {x.name: x for x in w}


def get(name: str) -> Workload:
    return workloads()[name]


def make_inputs(wl: Workload, device="cpu", generator_device: Optional[str] = None):
    """Draw the workload's tensors (contiguous, packed) on ``device``.

    Values are drawn with a torch generator seeded by ``wl.seed`` on
    ``generator_device`` (default: ``device``) in fp32, scaled by ``wl.std``
    and rounded to ``wl.dtype``.  Returns a dict with q, q_rope, k, k_rope, v
    (16-bit) and q_seqlen, kv_seqlen (int32, on ``device``).
    """
    gdev = torch.device(generator_device or device)
    gen = torch.Generator(device=gdev)
    gen.manual_seed(wl.seed)
    H, G, Dn, R = wl.head_num, wl.kv_head_num, wl.d_nope, wl.d_rope

    def draw(*shape):
        x = torch.randn(*shape, generator=gen, device=gdev, dtype=torch.float32)
        if wl.std != 1.0:
            x.mul_(wl.std)
        return x.to(wl.dtype).to(device)

    out = {
        "q": draw(wl.t_q, H, Dn),
        "q_rope": draw(wl.t_q, H, R),
        "k": draw(wl.t_k, G, Dn),
        "k_rope": draw(wl.t_k, G, R),
        "v": draw(wl.t_k, G, Dn),
        "q_seqlen": torch.tensor(wl.q_seqlens, dtype=torch.int32, device=device),
        "kv_seqlen": torch.tensor(wl.kv_seqlens, dtype=torch.int32, device=device),
    }
    return out


def sample_rows(seq_len: int, n: int, seed: int) -> np.ndarray:
    """Seeded query rows of one sequence for sampled checks.

    Always includes the tile-edge rows {0, 1, 127, 128, 129, 255, 256, L-129,
    L-128, L-1} (those < L), then fills up to n with distinct rows drawn by
    numpy default_rng(seed).
    """
    fixed = [0, 1, 127, 128, 129, 255, 256, seq_len - 129, seq_len - 128, seq_len - 1]
    fixed = sorted({r for r in fixed if 0 <= r < seq_len})
    rest = np.setdiff1d(np.arange(seq_len), fixed)
    k = max(0, min(n - len(fixed), rest.size))
    drawn = np.random.default_rng(seed).choice(rest, size=k, replace=False) if k else np.array([], dtype=np.int64)
    return np.sort(np.concatenate([np.asarray(fixed, dtype=np.int64), drawn.astype(np.int64)]))


def paged_cache(k, k_rope, v, kv_seqlens, block_size, seed=7, spare_blocks=0, slot_fill=0.0, table_fill=-1):
    """Scatters packed keys / values into a block-paged cache (the ND keyCache / valueCache
    layout of the PagedCacheLoadOperation page), blocks handed out in a seeded random order.

    Returns (key_cache [blocks, block_size, G, 192] holding K_nope | K_rope per slot,
    value_cache [blocks, block_size, G, 128], block_tables [batch, W] int32).  Slots no key
    occupies (the tail of each sequence's last block, the spare blocks) hold `slot_fill`; table
    entries past a sequence's last block hold `table_fill`.  Pure data movement.
    """
    device = k.device
    G = k.shape[1]
    kcat = torch.cat([k, k_rope], dim=2)
    need = [(L + block_size - 1) // block_size for L in kv_seqlens]
    nb = sum(need) + spare_blocks
    perm = torch.randperm(max(nb, 1), generator=torch.Generator().manual_seed(seed))[:nb]
    kc = torch.full((max(nb, 1), block_size, G, kcat.shape[2]), slot_fill, dtype=k.dtype, device=device)
    vc = torch.full((max(nb, 1), block_size, G, v.shape[2]), slot_fill, dtype=v.dtype, device=device)
    table = torch.full((len(need), max(need + [1])), table_fill, dtype=torch.int32)
    used = start = 0
    for b, L in enumerate(kv_seqlens):
        n = need[b]
        if n:
            idx = perm[used:used + n]
            table[b, :n] = idx.to(torch.int32)
            full = L // block_size
            dev_idx = idx.to(device)
            if full:
                kc[dev_idx[:full]] = kcat[start:start + full * block_size].view(full, block_size, G, -1)
                vc[dev_idx[:full]] = v[start:start + full * block_size].view(full, block_size, G, -1)
            rem = L - full * block_size
            if rem:
                kc[int(idx[full]), :rem] = kcat[start + full * block_size:start + L]
                vc[int(idx[full]), :rem] = v[start + full * block_size:start + L]
        used += n
        start += L
    return kc, vc, table.to(device)


@dataclass
class PrologShape:
    """Sizes of the MlaProlog step (the page's supported configuration by default:
    h 4096, q_lora_rank 1024, 64 heads of head_dim 512, rope_dim 64)."""
    name: str
    tokens: int
    hidden: int = 4096
    q_lora_rank: int = 1024
    num_heads: int = 64
    head_dim: int = 512
    rope_dim: int = 64
    seed: int = 6


def prolog_shapes() -> dict:
    return {s.name: s for s in [
        PrologShape("prolog_small", tokens=77, hidden=512, q_lora_rank=256, num_heads=4, head_dim=256,
                    rope_dim=64, seed=61),
        PrologShape("prolog", tokens=4096),
    ]}


def make_prolog_inputs(s: PrologShape, device="cpu", positions=None):
    """Synthetic bf16 inputs of the MlaProlog step on ``device``.

    token_x ~ N(0, 1); projection weights ~ N(0, 1 / fan_in) (random init, no trained weights);
    RmsNorm weights 1 + 0.25 N(0, 1); rope_cos / rope_sin for token positions (default
    0 .. tokens-1) at angles pos * 10000^(-2i / rope_dim), each value repeated for the two
    channels of its interleaved pair.  Drawn in fp32 with a seeded CPU generator, rounded to bf16.
    """
    gen = torch.Generator().manual_seed(s.seed)

    def draw(*shape, scale=1.0, shift=0.0):
        return (torch.randn(*shape, generator=gen) * scale + shift).to(torch.bfloat16).to(device)

    t, h, r, d = s.tokens, s.hidden, s.q_lora_rank, s.head_dim
    pos = torch.arange(t, dtype=torch.float64) if positions is None else torch.as_tensor(positions, dtype=torch.float64)
    inv = 10000.0 ** (-torch.arange(0, s.rope_dim, 2, dtype=torch.float64) / s.rope_dim)
    ang = pos[:, None] * inv[None, :]
    return {
        "token_x": draw(t, h),
        "wq_a": draw(h, r, scale=h ** -0.5),
        "wq_b": draw(r, s.num_heads * d, scale=r ** -0.5),
        "wkv": draw(h, d, scale=h ** -0.5),
        "rope_cos": torch.cos(ang).repeat_interleave(2, dim=1).to(torch.bfloat16).to(device),
        "rope_sin": torch.sin(ang).repeat_interleave(2, dim=1).to(torch.bfloat16).to(device),
        "gamma_cq": draw(r, scale=0.25, shift=1.0),
        "gamma_ckv": draw(d, scale=0.25, shift=1.0),
    }
