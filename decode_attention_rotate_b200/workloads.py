"""Seeded synthetic workloads for the 2-bit rotated MLA cache.

This module only draws inputs: shapes, seeds and value distributions.  It holds none
of the method's arithmetic (no rotation, quantisation or attention), so both the CPU
oracle and the CUDA path can take their inputs from it.

Distributions (one request's cache is a DeepSeek-V2-Lite-shaped MLA layer: a 512-d
content latent and a 64-d RoPE key per token, "RoLaQ", §2.1 and §A.3):
  * content latent c ~ N(0, sigma_ch^2), sigma_ch ~ lognormal(0, 0.5) drawn once per
    channel and layer;
  * RoPE key k_R ~ N(0, 1) with 6 fixed outlier channels scaled by 10 (about a tenth
    of the 64 channels carry outliers, as the RAQ-MLA review's k_R analysis reports);
  * queries: q_c_rot ~ N(0, 1) and q_R ~ N(0, 1) in bf16.  For an orthogonal R and
    q_c ~ N(0, I), q_c . R is again N(0, I), so drawing the rotated query directly has
    the distribution of folding R into the query;
  * R: Q factor of a seeded N(0, 1) 512x512 matrix with the diagonal of the triangular
    factor made positive, stored fp32;
  * per-layer tau ~ U[0.85, 1.1] and gain ~ U[1.0, 1.2] (the tiny case fixes
    tau = 0.9816 and gain = 1.16).
All values that end in bf16 are rounded to nearest-even by torch.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

D_C = 512
D_R = 64
PAGE_TOKENS = 64
N_OUTLIER = 6
OUTLIER_SCALE = 10.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq_lens: tuple          # per request
    heads: int
    layers: int = 1
    tau: Optional[float] = None   # None: drawn per layer
    gain: Optional[float] = None
    paged_shuffled: bool = False
    n_sink: int = 0
    n_recent: int = 0
    seed: int = 1000

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    def pages_per_seq(self) -> List[int]:
        return [(L + PAGE_TOKENS - 1) // PAGE_TOKENS for L in self.seq_lens]


def _loguniform_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(round(math.exp(x))) for x in u)


# The five workloads.  Sizes follow the serving shapes: a tiny single-layer check,
# a 4 x 32K one-layer decode, 4 x 256K over 27 layers, a 128-head paged batch with
# log-uniform lengths, and a 64K-token prefill + 64 x 8K decode with 4 sink and 128
# recent BF16 tokens.
TINY = Workload("tiny_1x256_h16", 1, (256,), 16, tau=0.9816, gain=1.16, seed=1000)
DECODE_4x32K = Workload("decode_4x32k_h16", 4, (32768,) * 4, 16, seed=1001)
DECODE_4x256K_27L = Workload("decode_4x256k_h16_27layers", 4, (262144,) * 4, 16,
                             layers=27, seed=1002)
PAGED_H128 = Workload("paged_h128_b32_1k_64k", 32,
                      _loguniform_lengths(1003, 32, 1024, 65536), 128,
                      paged_shuffled=True, seed=1003)
PREFILL_64K_27L = Workload("prefill_64k_27layers", 1, (65536,), 16, layers=27, seed=1004)
MIXED_64x8K = Workload("mixed_64x8k_sink4_recent128", 64, (8192,) * 64, 16,
                       n_sink=4, n_recent=128, seed=1005)

ALL = [TINY, DECODE_4x32K, DECODE_4x256K_27L, PAGED_H128, PREFILL_64K_27L, MIXED_64x8K]


def rng_for(w: Workload, layer: int = 0, stream: int = 0) -> np.random.Generator:
    return np.random.default_rng([w.seed, layer, stream])


def rotation(seed: int) -> np.ndarray:
    """Seeded orthogonal 512x512 fp32 matrix (Q of a Gaussian QR, sign-fixed)."""
    g = np.random.default_rng([seed, 77]).standard_normal((D_C, D_C))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return q.astype(np.float32)


def layer_constants(w: Workload, layer: int) -> tuple:
    """(tau, gain) for one layer."""
    if w.tau is not None:
        return float(w.tau), float(w.gain)
    rng = rng_for(w, layer, 9)
    return float(rng.uniform(0.85, 1.1)), float(rng.uniform(1.0, 1.2))


def channel_std(w: Workload, layer: int) -> np.ndarray:
    return rng_for(w, layer, 1).lognormal(0.0, 0.5, size=D_C)


def outlier_channels(w: Workload) -> np.ndarray:
    return np.sort(np.random.default_rng([w.seed, 5]).choice(D_R, N_OUTLIER, replace=False))


def to_bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def latent(w: Workload, layer: int, n_tokens: int, stream: int = 2) -> torch.Tensor:
    """bf16 content latents [n_tokens, 512] (CPU)."""
    rng = rng_for(w, layer, stream)
    std = channel_std(w, layer)
    return to_bf16(rng.standard_normal((n_tokens, D_C)) * std[None, :])


def rope_key(w: Workload, layer: int, n_tokens: int, stream: int = 3) -> torch.Tensor:
    rng = rng_for(w, layer, stream)
    k = rng.standard_normal((n_tokens, D_R))
    k[:, outlier_channels(w)] *= OUTLIER_SCALE
    return to_bf16(k)


def queries(w: Workload, layer: int, stream: int = 4):
    """(q_c_rot [B,H,512], q_R [B,H,64]) bf16 (CPU)."""
    rng = rng_for(w, layer, stream)
    q_c = rng.standard_normal((w.batch, w.heads, D_C))
    q_r = rng.standard_normal((w.batch, w.heads, D_R))
    return to_bf16(q_c), to_bf16(q_r)


def page_table(w: Workload, max_pages: Optional[int] = None) -> np.ndarray:
    """int32 [batch, max_pages]; contiguous per request unless paged_shuffled, in which
    case the pool's pages are handed out in a seeded random order.  Unused entries -1."""
    pps = w.pages_per_seq()
    mp = max(pps) if max_pages is None else max_pages
    total = sum(pps)
    order = np.arange(total, dtype=np.int64)
    if w.paged_shuffled:
        order = np.random.default_rng([w.seed, 6]).permutation(total)
    pt = np.full((w.batch, mp), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(pps):
        pt[b, :n] = order[k:k + n]
        k += n
    return pt


# ---- device-side generators for the large workloads ---------------------------------

def device_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def latent_device(w: Workload, layer: int, n_tokens: int, device, stream: int = 2) -> torch.Tensor:
    g = device_generator(w.seed * 1000003 + layer * 101 + stream, device)
    std = torch.as_tensor(channel_std(w, layer), dtype=torch.float32, device=device)
    x = torch.randn((n_tokens, D_C), generator=g, device=device, dtype=torch.float32)
    return (x * std[None, :]).to(torch.bfloat16)


def rope_key_device(w: Workload, layer: int, n_tokens: int, device, stream: int = 3) -> torch.Tensor:
    g = device_generator(w.seed * 1000003 + layer * 101 + stream, device)
    k = torch.randn((n_tokens, D_R), generator=g, device=device, dtype=torch.float32)
    idx = torch.as_tensor(outlier_channels(w), device=device)
    k[:, idx] *= OUTLIER_SCALE
    return k.to(torch.bfloat16)
