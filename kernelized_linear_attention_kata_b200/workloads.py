"""Seeded synthetic inputs for the KATA forward and decode workloads.

This module only draws random numbers and shapes them (unit-normalising rows,
projecting hidden states, picking pool entries). It holds none of the
method's arithmetic, so that the CUDA path and the test oracle can both take
their inputs from it without sharing any computation.

Every generator returns tensors already rounded to the workload's dtype; the
oracle widens exactly these values to float64.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

PSD = "psd"
FIRST_ORDER = "first_order"


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d_k: int
    d_v: int
    C: int
    dtype: str            # "f32" or "bf16": element type of q, k, v and the output
    feature: str          # "psd" or "first_order"
    seed: int
    recipe: str           # "unit", "projected" or "mqar"
    v_std: float = 1.0
    width: int = 0        # model width for the "projected" recipe

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T)


# The five workloads. Sizes follow the problem statement of the pages (Q, K, V
# [B, H, T, d], chunk size C); the recipes are stated in the design notes.
TINY = Workload("tiny_f32", B=1, H=1, T=256, d_k=16, d_v=16, C=64, dtype="f32",
                feature=PSD, seed=1, recipe="unit")
MID = Workload("mid_bf16", B=4, H=8, T=4096, d_k=32, d_v=64, C=64, dtype="bf16",
               feature=PSD, seed=2, recipe="unit", v_std=0.5)
LAYER = Workload("layer340m_bf16", B=8, H=16, T=2048, d_k=32, d_v=64, C=64, dtype="bf16",
                 feature=PSD, seed=3, recipe="projected", width=1024)
LONG = Workload("long131k_bf16", B=1, H=16, T=131072, d_k=32, d_v=64, C=128, dtype="bf16",
                feature=PSD, seed=4, recipe="mqar")
FIRST = Workload("first_order64k_bf16", B=2, H=16, T=65536, d_k=64, d_v=64, C=64, dtype="bf16",
                 feature=FIRST_ORDER, seed=5, recipe="unit")
WORKLOADS = {w.name: w for w in (TINY, MID, LAYER, LONG, FIRST)}

# Quadratic-form comparison on the long workload: its first 16384 tokens.
LONG_QUADRATIC_T = 16384

# Batched decode: batch 256 x 16 heads, PSD state of d_k = 32, d_v = 64,
# prior state accumulated from 4096 seeded tokens per head.
DECODE_BATCH = 256
DECODE_HEADS = 16
DECODE_DK = 32
DECODE_DV = 64
DECODE_PRIOR_TOKENS = 4096
DECODE_SEED = 6


def _generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def unit_rows(x: torch.Tensor) -> torch.Tensor:
    """Rows divided by their L2 norm (the 'unit-normalised N(0,1)' recipe)."""
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def make_inputs(w: Workload, device="cpu"):
    """(q, k, v) for a workload, each [B, H, T, d] in the workload dtype."""
    g = _generator(w.seed, device)
    B, H, T = w.B, w.H, w.T
    if w.recipe == "unit":
        q = unit_rows(_randn((B, H, T, w.d_k), g, device))
        k = unit_rows(_randn((B, H, T, w.d_k), g, device))
        v = _randn((B, H, T, w.d_v), g, device) * w.v_std
    elif w.recipe == "projected":
        # Random-init projections (std 0.02) of N(0,1) hidden states; keys
        # unit-normalised, queries left raw.
        x = _randn((B, T, w.width), g, device)
        wq = _randn((w.width, H * w.d_k), g, device) * 0.02
        wk = _randn((w.width, H * w.d_k), g, device) * 0.02
        wv = _randn((w.width, H * w.d_v), g, device) * 0.02
        q = (x @ wq).view(B, T, H, w.d_k).permute(0, 2, 1, 3)
        k = unit_rows((x @ wk).view(B, T, H, w.d_k).permute(0, 2, 1, 3))
        v = (x @ wv).view(B, T, H, w.d_v).permute(0, 2, 1, 3)
    elif w.recipe == "mqar":
        # Per head: a pool of 256 unit keys, each bound to a fixed N(0,1)
        # value. Each position is a pool token with probability 1/2 (uniform
        # pool id; key and value taken from the pool) or a noise token (fresh
        # unit key, fresh N(0,1) value). Queries are fresh unit vectors.
        pool = 256
        q = unit_rows(_randn((B, H, T, w.d_k), g, device))
        keys_pool = unit_rows(_randn((B, H, pool, w.d_k), g, device))
        vals_pool = _randn((B, H, pool, w.d_v), g, device)
        noise_k = unit_rows(_randn((B, H, T, w.d_k), g, device))
        noise_v = _randn((B, H, T, w.d_v), g, device)
        is_pool = torch.rand((B, H, T), generator=g, device=device) < 0.5
        ids = torch.randint(0, pool, (B, H, T), generator=g, device=device)
        kp = torch.gather(keys_pool, 2, ids[..., None].expand(B, H, T, w.d_k))
        vp = torch.gather(vals_pool, 2, ids[..., None].expand(B, H, T, w.d_v))
        k = torch.where(is_pool[..., None], kp, noise_k)
        v = torch.where(is_pool[..., None], vp, noise_v)
    else:
        raise ValueError(w.recipe)
    dt = w.torch_dtype
    return (q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous())


def make_grad_output(w: Workload, device="cpu"):
    """Upstream gradient dL/dy for the backward, [B, H, T, d_v] N(0,1) in the
    workload dtype, seeded apart from the inputs."""
    g = _generator(w.seed + 7919, device)
    return _randn((w.B, w.H, w.T, w.d_v), g, device).to(w.torch_dtype).contiguous()


def make_decode_inputs(batch=DECODE_BATCH, heads=DECODE_HEADS, d_k=DECODE_DK, d_v=DECODE_DV,
                       seed=DECODE_SEED, device="cpu", dtype=torch.bfloat16):
    """The decode step's token: q, k unit [batch, H, d_k]; v N(0,1) [batch, H, d_v]."""
    g = _generator(seed, device)
    q = unit_rows(_randn((batch, heads, d_k), g, device))
    k = unit_rows(_randn((batch, heads, d_k), g, device))
    v = _randn((batch, heads, d_v), g, device)
    return q.to(dtype).contiguous(), k.to(dtype).contiguous(), v.to(dtype).contiguous()


def make_decode_prior_tokens(batch, heads, n_tokens=DECODE_PRIOR_TOKENS, d_k=DECODE_DK,
                             d_v=DECODE_DV, seed=DECODE_SEED + 1000, device="cpu",
                             dtype=torch.bfloat16):
    """Seeded prior tokens (k unit, v N(0,1)), [batch, H, n_tokens, d], from
    which each side builds the decode step's prior state (S, z)."""
    g = _generator(seed, device)
    k = unit_rows(_randn((batch, heads, n_tokens, d_k), g, device))
    v = _randn((batch, heads, n_tokens, d_v), g, device)
    return k.to(dtype).contiguous(), v.to(dtype).contiguous()


def to_f64_numpy(t: torch.Tensor):
    """Exact widening of the rounded inputs for the oracle."""
    return t.detach().to("cpu", torch.float64).numpy()


def make_delta_beta(B, H, T, seed, device="cpu"):
    """DeltaKATA write strengths [B, H, T] fp32: uniform in (0, 1], with
    every fourth token at exactly 1 (a full overwrite)."""
    g = _generator(seed + 313, device)
    u = torch.rand((B, H, T), generator=g, device=device, dtype=torch.float32)
    beta = 1.0 - u * 0.9                      # (0.1, 1]
    beta[..., ::4] = 1.0
    return beta.contiguous()
