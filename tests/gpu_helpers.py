"""Helpers shared by the GPU parity tests: move oracle-built caches to the device, read
device caches back, and the comparison rules (codes, metadata, decode output)."""
import math

import numpy as np
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W

Z_WINDOW = 1e-5          # codes may differ only within this distance of a threshold
META_TOL = 1e-6          # metadata tolerance (relative; mean measured against |mean| + std)
DECODE_TOL = 1e-2        # relative L2 per (request, head)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def codes_match(gpu_packed, oracle_q, tau):
    """Bit-exact codes except coordinates whose oracle z lies within Z_WINDOW of -tau, 0
    or tau.  Returns (ok, fraction_in_window, n_mismatch_outside)."""
    g = O.unpack(gpu_packed)
    o = oracle_q["codes"]
    z = oracle_q["z"]
    near = (np.abs(z - tau) < Z_WINDOW) | (np.abs(z) < Z_WINDOW) | (np.abs(z + tau) < Z_WINDOW)
    bad = (g != o) & ~near
    return int(bad.sum()) == 0, float(near.mean()), int(bad.sum())


def meta_match(gpu_meta, oracle_q, gain):
    mu_o, sd_o = oracle_q["mu"], oracle_q["sd"]
    mu_g = gpu_meta[:, :, 0].astype(np.float64)
    s_g = gpu_meta[:, :, 1].astype(np.float64)
    s_o = gain * sd_o
    err_mu = np.abs(mu_g - mu_o) / (np.abs(mu_o) + sd_o + 1e-300)
    err_s = np.abs(s_g - s_o) / np.maximum(s_o, 1e-300)
    err_s = np.where(s_o == 0, np.abs(s_g), err_s)
    return float(err_mu.max()), float(err_s.max())


def rel_l2(a, b):
    num = np.sqrt(((a - b) ** 2).sum(axis=-1))
    den = np.sqrt((b ** 2).sum(axis=-1))
    return num / np.maximum(den, 1e-300)


def build_oracle_cache(w: W.Workload, layer: int, seq_lens, tau, gain, n_sink=0, n_recent=0,
                       device="cuda"):
    """Quantize every request on the CPU oracle and lay the records out in pages.
    Returns (PagedCache on device, per-request dict of oracle data)."""
    Rm = W.rotation(w.seed + layer).astype(np.float64)
    pt = W.page_table(W.Workload(w.name, len(seq_lens), tuple(seq_lens), w.heads,
                                 paged_shuffled=w.paged_shuffled, seed=w.seed))
    num_pages = int(max(pt.max() + 1, 1))
    pool = np.zeros(num_pages * O.PAGE_BYTES, np.uint8)
    data = []
    for r, L in enumerate(seq_lens):
        c = W.latent(w, layer, L, stream=100 + r)
        kr = W.rope_key(w, layer, L, stream=200 + r)
        q = O.quantize(f64(c), Rm, tau, gain)
        kr_bits = bf16_bits(kr)
        if L:
            O.pages_write(pool, pt, r, q["packed"], q["meta"], kr_bits)
        data.append({"q": q, "k_r": f64(kr), "y": q["y"]})
    cache = R.PagedCache(num_pages, torch.as_tensor(pt), n_sink, n_recent, device=device,
                         pages=torch.as_tensor(pool).to(device))
    if cache.prot is not None:
        nslot = n_sink + n_recent
        prot = np.zeros((len(seq_lens), nslot, O.D_C), np.float64)
        for r, L in enumerate(seq_lens):
            yb = O.bf16_round(data[r]["y"])
            for p in range(L):
                if p < n_sink:
                    prot[r, p] = yb[p]
                elif p >= L - n_recent:
                    prot[r, n_sink + p % n_recent] = yb[p]
        cache.prot.copy_(torch.as_tensor(prot, dtype=torch.float32).to(torch.bfloat16))
        for r, L in enumerate(seq_lens):
            data[r]["prot_content"] = O.bf16_round(data[r]["y"])
    return cache, data, Rm


def oracle_decode(data, q_c, q_r, seq_lens, tau, sm_scale, n_sink=0, n_recent=0):
    B, H = q_c.shape[0], q_c.shape[1]
    out = np.zeros((B, H, O.D_C))
    lse = np.zeros((B, H))
    for r, L in enumerate(seq_lens):
        d = data[r]
        o, l = O.decode_request(q_c[r], q_r[r], d["q"]["packed"], d["q"]["meta"], d["k_r"], tau,
                                sm_scale, d.get("prot_content"), n_sink, n_recent)
        out[r], lse[r] = o, l
    return out, lse


SM_SCALE = 1.0 / math.sqrt(192.0)
