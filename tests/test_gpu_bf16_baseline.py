"""The BF16 comparison point of the benchmark (a library kernel, FlashInfer's MLA decode on
an uncompressed bf16 cache) computes the same absorbed-MLA decode as the oracle with
quantisation switched off, so the time ratio the benchmark reports compares like with
like.  Skipped when FlashInfer is not installed."""
import math

import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_bf16_library_decode_matches_oracle_without_quantisation():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    fi_mla = pytest.importorskip("flashinfer.mla")
    w = W.Workload("bf16ref", 3, (700, 64, 1500), 16, seed=909)
    page = 64
    npg = [(L + page - 1) // page for L in w.seq_lens]
    mp = max(npg)
    kv = torch.zeros((sum(npg), page, 576), dtype=torch.bfloat16)
    bt = torch.zeros((w.batch, mp), dtype=torch.int32)
    xs, krs = [], []
    k0 = 0
    for b, L in enumerate(w.seq_lens):
        x = W.latent(w, 0, L, stream=10 + b)            # bf16 latent, taken as stored content
        kr = W.rope_key(w, 0, L, stream=20 + b)
        flat = torch.cat([x, kr], dim=1)
        rows = torch.zeros((npg[b] * page, 576), dtype=torch.bfloat16)
        rows[:L] = flat
        kv[k0:k0 + npg[b]] = rows.reshape(npg[b], page, 576)
        bt[b, :npg[b]] = torch.arange(k0, k0 + npg[b], dtype=torch.int32)
        k0 += npg[b]
        xs.append(x)
        krs.append(kr)
    q_c, q_r = W.queries(w, 0)
    q = torch.cat([q_c, q_r], dim=2).unsqueeze(1)      # [B, 1, H, 576]
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32)
    ws = torch.zeros(128 * 1024 * 1024, dtype=torch.uint8, device=DEV)
    sm = 1.0 / math.sqrt(192.0)
    out = fi_mla.trtllm_batch_decode_with_kv_cache_mla(
        q.to(DEV), kv.to(DEV), ws, 128, 512, 64, bt.to(DEV), lens.to(DEV), max(w.seq_lens),
        bmm1_scale=sm, bmm2_scale=1.0)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64).reshape(w.batch, w.heads, 512)
    for b in range(w.batch):
        ref, _ = O.attend(q_c[b].float().numpy(), q_r[b].float().numpy(),
                          xs[b].float().numpy().astype(np.float64), krs[b].float().numpy(), sm)
        err = np.sqrt(((got[b] - ref) ** 2).sum(-1)) / np.sqrt((ref ** 2).sum(-1))
        assert err.max() <= 1e-2, (b, float(err.max()))
