"""Seeded synthetic inputs shaped like the Wan2.2 workloads of the HiF4 path.

This module only draws random numbers and lays them out; it holds none of
the HiF4 arithmetic.  Both the CUDA path's tests/benchmark and the CPU oracle
consume exactly the bytes produced here (numpy ``default_rng(seed)``, PCG64;
BF16 by round-to-nearest-even from float32).  A device-side variant using a
seeded ``torch.Generator`` serves the largest benchmark tensors, where host
generation would take minutes; the oracle then reads back sampled rows.

Workloads (seed, shape, distribution):

1. ``tiny``  (seed 0): X fp32 128x512 ~ N(0,1) with 327 distinct seeded
   positions (0.5 % of the entries) multiplied by 50; W fp32 512x512 ~ N(0, 0.02^2).
2. ``quant_sweep`` (seed 1): n BF16 values laid out as rows of 5120 (the last
   row partial); x = t_3 * 0.05 * s_row, s_row ~ LogNormal(0, 1).
3. ``attn_proj`` (seed 2): X bf16 M x 5120 = N(0,1) * sigma_c,
   sigma_c ~ LogNormal(0, 0.5), 51 seeded channels with sigma x20 (these are
   the protected channels); W bf16 5120x5120 ~ N(0, 0.015^2); bias ~ N(0, 0.01^2).
   M = 57600 = 16 latent frames x 3600 tokens.
4. ``ffn`` (seed 3): X as in 3; W1 13824x5120, W2 5120x13824 ~ N(0, 0.015^2);
   no bias.  A GELU-shaped stand-in for the hidden activation H (positive
   part of N(0,1)*sigma_c plus a 0.1-scaled negative part) for testing the
   second linear on its own.
5. ``calib`` (seed 4): T = 16 x 14400 tokens x C = 5120 channels, N(0, sigma_c^2),
   sigma_c ~ LogNormal(0, 0.5); 102 seeded spike channels in which each entry
   is multiplied by 100 with probability 1e-4.
"""
from __future__ import annotations

import math

import numpy as np

WAN_TOKENS = 57600          # 16 latent frames x 3600 tokens
WAN_DIM = 5120
WAN_FFN = 13824
CALIB_TOKENS = 16 * 14400
_ROW = 5120


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------- workload 1

def tiny(seed: int = 0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((128, 512)).astype(np.float32)
    n_out = int(0.005 * X.size)                   # 327
    pos = rng.choice(X.size, size=n_out, replace=False)
    X.reshape(-1)[pos] *= np.float32(50.0)
    W = (rng.standard_normal((512, 512)) * 0.02).astype(np.float32)
    return X, W


# --------------------------------------------------------------- workload 2

def quant_sweep(n: int, seed: int = 1, chunk: int = 1 << 22) -> np.ndarray:
    """n BF16 values (uint16 bit patterns, flat)."""
    rng = np.random.default_rng(seed)
    nrows = -(-n // _ROW)
    s_row = rng.lognormal(0.0, 1.0, size=nrows)
    out = np.empty(n, np.uint16)
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        t = rng.standard_t(3, size=b - a)
        rows = np.arange(a, b) // _ROW
        out[a:b] = f32_to_bf16_bits((t * 0.05 * s_row[rows]).astype(np.float32))
    return out


def quant_sweep_torch(n: int, device, seed: int = 1):
    """Device-side variant of workload 2 for the largest sizes (torch RNG)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    nrows = -(-n // _ROW)
    s_row = torch.empty(nrows, device=device).log_normal_(0.0, 1.0, generator=g)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    chunk = 1 << 26
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        z = torch.randn(b - a, device=device, generator=g)
        chi = torch.randn(3, b - a, device=device, generator=g).square_().sum(0).div_(3.0)
        t = z / chi.sqrt_()
        rows = torch.arange(a, b, device=device) // _ROW
        out[a:b] = (t * 0.05 * s_row[rows]).to(torch.bfloat16)
    return out


# --------------------------------------------------------------- workload 3/4

def _channel_sigmas(rng, C: int, n_outlier: int):
    sigma = rng.lognormal(0.0, 0.5, size=C)
    outl = np.sort(rng.choice(C, size=n_outlier, replace=False)).astype(np.int32)
    sigma[outl] *= 20.0
    return sigma.astype(np.float32), outl


def _rows(rng, M: int, sigma: np.ndarray, chunk_rows: int = 2048) -> np.ndarray:
    C = sigma.size
    out = np.empty((M, C), np.uint16)
    for a in range(0, M, chunk_rows):
        b = min(M, a + chunk_rows)
        z = rng.standard_normal((b - a, C), dtype=np.float32)
        out[a:b] = f32_to_bf16_bits(z * sigma)
    return out


def attn_proj(M: int = WAN_TOKENS, K: int = WAN_DIM, N: int = WAN_DIM, seed: int = 2):
    """-> dict(x, w, bias, mask_idx) with BF16 bit patterns (uint16)."""
    rng = np.random.default_rng(seed)
    sigma, outl = _channel_sigmas(rng, K, max(1, K // 100))
    w = f32_to_bf16_bits((rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.015)))
    bias = f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))
    x = _rows(rng, M, sigma)
    return dict(x=x, w=w, bias=bias, mask_idx=outl)


def ffn(M: int = WAN_TOKENS, D: int = WAN_DIM, F: int = WAN_FFN, seed: int = 3,
        with_x: bool = True):
    """-> dict(x, w1, w2) BF16 bit patterns; x may be skipped (with_x=False)."""
    rng = np.random.default_rng(seed)
    sigma, _ = _channel_sigmas(rng, D, max(1, D // 100))
    w1 = f32_to_bf16_bits(rng.standard_normal((F, D), dtype=np.float32) * np.float32(0.015))
    w2 = f32_to_bf16_bits(rng.standard_normal((D, F), dtype=np.float32) * np.float32(0.015))
    x = _rows(rng, M, sigma) if with_x else None
    return dict(x=x, w1=w1, w2=w2)


def ffn_hidden(M: int, F: int = WAN_FFN, seed: int = 33) -> np.ndarray:
    """GELU-shaped stand-in for the FFN hidden activation (BF16 bits)."""
    rng = np.random.default_rng(seed)
    sigma = rng.lognormal(0.0, 0.5, size=F).astype(np.float32)
    out = np.empty((M, F), np.uint16)
    for a in range(0, M, 1024):
        b = min(M, a + 1024)
        z = rng.standard_normal((b - a, F), dtype=np.float32) * sigma
        out[a:b] = f32_to_bf16_bits(np.where(z > 0, z, np.float32(0.1) * z))
    return out


def device_rows(M: int, C: int, seed: int, device, n_outlier: int | None = None):
    """Device-side X like workload 3 (torch RNG), BF16 tensor M x C."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sigma = torch.empty(C, device=device).log_normal_(0.0, 0.5, generator=g)
    k = max(1, C // 100) if n_outlier is None else n_outlier
    outl = torch.randperm(C, device=device, generator=g)[:k].sort().values.to(torch.int32)
    sigma[outl.long()] *= 20.0
    x = torch.empty(M, C, dtype=torch.bfloat16, device=device)
    for a in range(0, M, 4096):
        b = min(M, a + 4096)
        x[a:b] = (torch.randn(b - a, C, device=device, generator=g) * sigma).to(torch.bfloat16)
    return x, outl


def device_weight(N: int, K: int, std: float, seed: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return (torch.randn(N, K, device=device, generator=g) * std).to(torch.bfloat16)


# --------------------------------------------------------------- workload 5

def calib(T: int = CALIB_TOKENS, C: int = WAN_DIM, seed: int = 4,
          spike_frac: float = 0.02, spike_p: float = 1e-4, spike_mul: float = 100.0):
    """-> (acts uint16 T x C BF16 bits, spike_channels int32)."""
    rng = np.random.default_rng(seed)
    sigma = rng.lognormal(0.0, 0.5, size=C).astype(np.float32)
    spikes = np.sort(rng.choice(C, size=int(spike_frac * C), replace=False)).astype(np.int32)
    is_spike = np.zeros(C, bool)
    is_spike[spikes] = True
    out = np.empty((T, C), np.uint16)
    for a in range(0, T, 2048):
        b = min(T, a + 2048)
        z = rng.standard_normal((b - a, C), dtype=np.float32) * sigma
        hit = (rng.random((b - a, C), dtype=np.float32) < np.float32(spike_p)) & is_spike
        z[hit] *= np.float32(spike_mul)
        out[a:b] = f32_to_bf16_bits(z)
    return out, spikes


def calib_torch(T: int, C: int, device, seed: int = 4, spike_frac: float = 0.02,
                spike_p: float = 1e-4, spike_mul: float = 100.0):
    """Device-side variant of workload 5 (torch RNG) -> BF16 tensor T x C."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sigma = torch.empty(C, device=device).log_normal_(0.0, 0.5, generator=g)
    spikes = torch.randperm(C, device=device, generator=g)[: int(spike_frac * C)]
    is_spike = torch.zeros(C, dtype=torch.bool, device=device)
    is_spike[spikes] = True
    x = torch.empty(T, C, dtype=torch.bfloat16, device=device)
    for a in range(0, T, 8192):
        b = min(T, a + 8192)
        z = torch.randn(b - a, C, device=device, generator=g) * sigma
        hit = (torch.rand(b - a, C, device=device, generator=g) < spike_p) & is_spike
        z = torch.where(hit, z * spike_mul, z)
        x[a:b] = z.to(torch.bfloat16)
    return x


def rows_for(n: int, cols: int = 1024) -> tuple[int, int]:
    """View a flat n-element tensor as rows x cols (cols | n, cols % 64 == 0)."""
    assert n % cols == 0 and cols % 64 == 0
    return n // cols, cols


def sample_rows(M: int, n: int, seed: int = 1234) -> np.ndarray:
    """Seeded sorted sample of row indices (always includes the last row)."""
    if n >= M:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    s = rng.choice(M - 1, size=n - 1, replace=False)
    return np.sort(np.append(s, M - 1))


__all__ = [n for n in dir() if not n.startswith("_") and n != "math"]
