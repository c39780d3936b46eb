"""Seeded synthetic inputs for the rotated-token KV-cache quantizer.

This module holds only input generators: no step of the method is computed
here.  The same generators feed both the CUDA path and the CPU oracle, so
that the two see identical inputs.  Every draw is seeded; the shapes and
value distributions follow the workloads of the pages:

* head_dim 128, Llama-3-8B-shaped grouped-query attention (32 query heads,
  8 KV heads), contexts of 32k-128k tokens (TurboQuant blog, "O Gargalo do
  Cache KV" and "Beneficios": 32k-128k+ contexts);
* outlier channels and per-channel offsets in keys (NSNQuant summary,
  "As Letras Miudas": outliers survive in early layers);
* channel means and token-norm spread for the NSN front end (NSNQuant,
  section 1: tokens differ in norm, channels are off-centre).

All generators return torch tensors on the requested device; the random
streams are torch's (CPU: Mersenne Twister, CUDA: Philox), so a given test
draws on one device and copies to the other side.  Distributions use the
numpy convention N(mu, sigma) / lognormal(mu, sigma) with sigma the standard
deviation of the normal.
"""
from __future__ import annotations

import torch

HEAD_DIM = 128


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _randn(shape, g, device, dtype=torch.float32):
    return torch.randn(shape, generator=g, device=device, dtype=dtype)


def _lognormal(shape, sigma, g, device):
    return torch.exp(sigma * _randn(shape, g, device))


def gaussian(n: int, d: int, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """i.i.d. N(0, 1) rows (tiny reference workload: 4096 x 128 fp32, seed 0)."""
    g = _gen(seed, device)
    return _randn((n, d), g, device).to(dtype)


def llama_keys(heads: int, tokens: int, d: int, seed: int, device="cpu", dtype=torch.bfloat16,
               outliers: int = 2, outlier_gain: float = 20.0) -> torch.Tensor:
    """Keys of one Llama-3-8B-shaped layer, [heads, tokens, d].

    Per head: channel scales lognormal(0, 0.5), ``outliers`` fixed channels
    (drawn once from the seed) multiplied by ``outlier_gain``, channel offsets
    N(0, 2); entries N(0, 1) * scale + offset.
    """
    g = _gen(seed, device)
    scale = _lognormal((heads, 1, d), 0.5, g, device)
    offset = 2.0 * _randn((heads, 1, d), g, device)
    for h in range(heads):
        ch = torch.randperm(d, generator=g, device=device)[:outliers]
        scale[h, 0, ch] *= outlier_gain
    x = _randn((heads, tokens, d), g, device) * scale + offset
    return x.to(dtype)


def llama_values(heads: int, tokens: int, d: int, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """Values of one layer, [heads, tokens, d]: N(0, 1) * lognormal(0, 0.3) per channel."""
    g = _gen(seed, device)
    scale = _lognormal((heads, 1, d), 0.3, g, device)
    return (_randn((heads, tokens, d), g, device) * scale).to(dtype)


def nsn_tokens(heads: int, tokens: int, d: int, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """NSN workload, [heads, tokens, d]: (N(0,1) + mu_c) * s_t, mu_c ~ N(0, 3), s_t ~ lognormal(0, 0.7)."""
    g = _gen(seed, device)
    mu = 3.0 * _randn((heads, 1, d), g, device)
    s = _lognormal((heads, tokens, 1), 0.7, g, device)
    return ((_randn((heads, tokens, d), g, device) + mu) * s).to(dtype)


def sweep_tokens(n: int, d: int, seed: int, device="cpu", dtype=torch.bfloat16, frac_hot: float = 0.01,
                 hot_gain: float = 10.0) -> torch.Tensor:
    """Sweep workload, [n, d]: N(0, 1) with a seeded ``frac_hot`` of rows scaled by ``hot_gain``."""
    g = _gen(seed, device)
    x = _randn((n, d), g, device)
    hot = torch.rand((n, 1), generator=g, device=device) < frac_hot
    x = torch.where(hot, x * hot_gain, x)
    return x.to(dtype)


def queries(batch: int, heads: int, d: int, seed: int, device="cpu", dtype=torch.bfloat16,
            std: float = 1.0) -> torch.Tensor:
    """Decode queries, [batch, heads, d]: N(0, std^2)."""
    g = _gen(seed, device)
    return (std * _randn((batch, heads, d), g, device)).to(dtype)


TINY = dict(n=4096, d=128, b=2, qjl=True, data_seed=0, handle_seed=1, scale=128 ** -0.5)
LLAMA_LAYER = dict(heads=8, tokens=32768, d=128, b=2, qjl=True, handle_seed=1, k_seed=11, v_seed=12)
DECODE = dict(batch=16, hq=32, hkv=8, d=128, T=131072, b=2, qjl=True, handle_seed=1, q_seed=31,
              q_std=128 ** -0.5, scale=1.0)
NSN = dict(heads=8, tokens=65536, d=128, b=2, qjl=False, handle_seed=1, seed=41)
SWEEP = dict(n=1 << 20, bits=(1, 2, 3, 4), qjl=(True, False), dims=(64, 128, 256), hkv=8, T=131072,
             handle_seed=1, seed=51)


def cache_slice_seed(base: int, batch: int, head: int, kind: int) -> int:
    """Seed of the synthetic K (kind 0) or V (kind 1) of one (sequence, KV head) of the decode workload."""
    return (base * 1_000_003 + batch * 4099 + head * 257 + kind) & 0x7FFF_FFFF
