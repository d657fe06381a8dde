"""Seeded input generators (data only; see the package docstring).

Host-side generators use ``numpy.random.default_rng(seed)`` and return numpy arrays;
bf16 tensors are carried as their uint16 bit patterns (round-to-nearest-even from
float32). Device-side generators (for the full-size workloads, which are too large
to build on the host) use a seeded ``torch.Generator`` on the GPU; tests that check
them copy the generated *inputs* back to the host for the oracle.

Workload recipes (synthetic stand-ins for Llama-3-8B-shaped layers; no checkpoint or
dataset is involved):

* weights ``W_base ~ N(0, base_std)``; fine-tune delta ``~ N(0, delta_std)`` with
  exactly ``round(frac * numel)`` entries, drawn without replacement, multiplied by
  ``mult`` (outliers); ``W_fine = W_base + delta`` rounded to the storage type. The
  delta the method sees is therefore the difference of the *stored* weights.
* activations ``x ~ N(0, 1)``.
* tenant ids: truncated Zipf, ``P(k) ~ k^-s`` for ``k = 1..T``, id = ``k - 1``.
* random tenants (when a delta need not come from a compress run): uniform random
  sign words and scales ``0.001 * sqrt(2/pi) * exp(0.1 z)``, ``z ~ N(0, 1)``, stored
  as fp16 (the abs-mean of ``N(0, 0.001)`` with a little spread).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "LLAMA3_8B_PROJECTIONS", "LLAMA3_8B_FUSED",
    "bf16_bits",
    "bf16_bits_to_f32",
    "weight_pair",
    "tiny_config",
    "zipf_ids",
    "activations",
    "random_tenant",
    "device_weight_pair",
    "device_random_tenant",
    "device_activations",
    "device_zipf_ids",
]

# (name, d_out, d_in) of the seven linear projections of one Llama-3-8B decoder layer.
LLAMA3_8B_PROJECTIONS = (
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
)

# The same layer as serving engines apply it: projections that read the same input are
# stacked along d_out (q | k | v and gate | up), so a layer is 4 products instead of 7
# with identical rows, columns, weights and outputs.
LLAMA3_8B_FUSED = (
    ("qkv", 6144, 4096),
    ("o", 4096, 4096),
    ("gate_up", 28672, 4096),
    ("down", 4096, 14336),
)


def bf16_bits(a) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _outlier_delta(rng, shape, delta_std, frac, mult):
    d = rng.normal(0.0, delta_std, size=shape)
    n = int(np.prod(shape))
    k = int(round(frac * n))
    if k:
        idx = rng.choice(n, size=k, replace=False)
        d.reshape(-1)[idx] *= mult
    return d


def weight_pair(seed: int, d_out: int, d_in: int, dtype: str = "bf16", base_std=0.02,
                delta_std=0.001, outlier_frac=0.0005, outlier_mult=30.0):
    """One (W_base, W_fine) pair on the host. ``dtype`` is ``"f32"`` (float32 arrays)
    or ``"bf16"`` (uint16 bit patterns)."""
    rng = np.random.default_rng(seed)
    wb = rng.normal(0.0, base_std, size=(d_out, d_in)).astype(np.float32)
    d = _outlier_delta(rng, (d_out, d_in), delta_std, outlier_frac, outlier_mult)
    if dtype == "f32":
        return wb, (wb.astype(np.float64) + d).astype(np.float32)
    if dtype == "bf16":
        wb_b = bf16_bits(wb)
        wf_b = bf16_bits((bf16_bits_to_f32(wb_b).astype(np.float64) + d).astype(np.float32))
        return wb_b, wf_b
    raise ValueError(dtype)


def tiny_config():
    """The small end-to-end case: one 256x512 fp32 pair, W_base ~ N(0, 0.02), delta
    ~ N(0, 0.002) with 0.1% of entries x20, group 128 with a 3-sigma clip; four fp32
    tokens split over two tenants with ids [0, 1, 0, 1]. ``default_rng(0)`` draws, in
    this order, W_base, tenant 0's delta, its outlier positions and x;
    ``default_rng(1)`` draws tenant 1's delta and outlier positions."""
    d_out, d_in = 256, 512
    rng0 = np.random.default_rng(0)
    wb = rng0.normal(0.0, 0.02, size=(d_out, d_in)).astype(np.float32)
    d0 = _outlier_delta(rng0, (d_out, d_in), 0.002, 0.001, 20.0)
    x = rng0.normal(0.0, 1.0, size=(4, d_in)).astype(np.float32)
    rng1 = np.random.default_rng(1)
    d1 = _outlier_delta(rng1, (d_out, d_in), 0.002, 0.001, 20.0)
    wf0 = (wb.astype(np.float64) + d0).astype(np.float32)
    wf1 = (wb.astype(np.float64) + d1).astype(np.float32)
    return {
        "w_base": wb, "w_fine": [wf0, wf1], "x": x,
        "tenant_ids": np.array([0, 1, 0, 1], dtype=np.int32),
        "group_size": 128, "clip": True, "clip_k": 3.0,
    }


def zipf_ids(rng, batch: int, n_tenants: int, s: float = 1.1) -> np.ndarray:
    """``batch`` tenant ids drawn from a Zipf(s) law truncated to ``n_tenants``."""
    k = np.arange(1, n_tenants + 1, dtype=np.float64)
    p = k ** (-s)
    p /= p.sum()
    return rng.choice(n_tenants, size=batch, p=p).astype(np.int32)


def activations(rng, batch: int, d_in: int, dtype: str = "bf16"):
    x = rng.normal(0.0, 1.0, size=(batch, d_in)).astype(np.float32)
    return bf16_bits(x) if dtype == "bf16" else x


def random_tenant(rng, d_out: int, d_in: int, mode: int, group_size: int = 128,
                  scale_dtype: str = "f16"):
    """Uniform random sign words plus abs-mean-like scales (host)."""
    words = rng.integers(0, 2 ** 32, size=(d_out, d_in // 32), dtype=np.uint64).astype(np.uint32)
    if mode == 0:
        shape = (d_out, d_in // group_size)
    elif mode == 1:
        shape = (d_out,)
    elif mode == 2:
        shape = (d_in,)
    elif mode == 4:
        shape = (-(-d_out // group_size), d_in // group_size)
    else:
        shape = (1,)
    z = rng.normal(0.0, 1.0, size=shape)
    s = 0.001 * math.sqrt(2.0 / math.pi) * np.exp(0.1 * z)
    s = s.astype(np.float16) if scale_dtype == "f16" else s.astype(np.float32)
    return {"signs": words, "scales": s, "scale_dtype": scale_dtype, "mode": mode,
            "group_size": group_size}


# ----------------------------------------------------------------------------------
# device-side generators (torch; imported lazily so the host generators need no GPU)
# ----------------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def device_weight_pair(gen, d_out, d_in, base_std=0.02, delta_std=0.001,
                       outlier_frac=0.0005, outlier_mult=30.0, device="cuda"):
    """bf16 (W_base, W_fine) built on the device from a seeded torch.Generator."""
    torch = _torch()
    wb = (torch.randn((d_out, d_in), generator=gen, device=device) * base_std).to(torch.bfloat16)
    d = torch.randn((d_out, d_in), generator=gen, device=device) * delta_std
    n = d_out * d_in
    k = int(round(outlier_frac * n))
    if k:
        idx = torch.randperm(n, generator=gen, device=device)[:k]
        d.view(-1)[idx] *= outlier_mult
    wf = (wb.float() + d).to(torch.bfloat16)
    del d
    return wb, wf


def device_random_tenant(gen, d_out, d_in, mode, group_size=128, device="cuda"):
    """Random sign words (int32 storage of uint32 words) and fp16 scales on the device."""
    torch = _torch()
    words = torch.randint(-(2 ** 31), 2 ** 31 - 1, (d_out, d_in // 32), generator=gen,
                          device=device, dtype=torch.int32)
    if mode == 0:
        shape = (d_out, d_in // group_size)
    elif mode == 1:
        shape = (d_out,)
    elif mode == 2:
        shape = (d_in,)
    elif mode == 4:
        shape = (-(-d_out // group_size), d_in // group_size)
    else:
        shape = (1,)
    z = torch.randn(shape, generator=gen, device=device)
    s = (0.001 * math.sqrt(2.0 / math.pi) * torch.exp(0.1 * z)).to(torch.float16)
    return words, s


def device_activations(gen, batch, d_in, device="cuda"):
    torch = _torch()
    return torch.randn((batch, d_in), generator=gen, device=device).to(torch.bfloat16)


def device_zipf_ids(gen, batch, n_tenants, s=1.1, device="cuda"):
    torch = _torch()
    k = torch.arange(1, n_tenants + 1, dtype=torch.float64, device=device)
    p = k.pow(-s)
    p = p / p.sum()
    return torch.multinomial(p, batch, replacement=True, generator=gen).to(torch.int32)
