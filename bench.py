#!/usr/bin/env python
"""Benchmark of the 2-bit rotated MLA cache hot path on B200.

Step = one decode step of the long-context serving shape: for each of 27 layers, one call
that appends one new token per request (write path: rotate, quantize, pack) and runs the
absorbed-MLA decode over 4 requests x 262,144 cached tokens at 16 heads (read path).  The cache of a
step is 8.15 GB, far larger than L2, so no flush is needed between steps.  value = cache
GB/s over the whole step (all ranks; replicas are independent, weak scaling).
Also measured: the prefill write path on 65,536 tokens x 27 layers (tokens/s), and the
CPU oracle on a bounded sample (cpu_baseline).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_attention_rotate_b200 import rolaq as R          # noqa: E402
from decode_attention_rotate_b200 import workloads as W      # noqa: E402

METRIC = "2-bit MLA decode: cache GB/s & % HBM roofline; quantize-append tokens/s"
SM_SCALE = 1.0 / math.sqrt(192.0)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# DRAM bytes (read + write) of the decode kernel per launch of the bench workload, taken
# from one ncu capture of the 4 x 131,072-token case (dram__bytes_read.sum +
# dram__bytes_write.sum; the reads scale with the tokens, x2 here, the split-K partials
# depend only on the item count, which is the same), together with the SHA-256 of the
# decode kernel sources it was taken on.  The bench reports it only while those sources
# are unchanged, and null otherwise.
DECODE_TRAFFIC = {"sources_sha256": "e319307d1b2c7dd94a8382c5694fce4dc0453f2b0108b4b0c1d5b9b7c63cd663",
                  "bytes_per_launch": 2 * 151.182848e6 + 4.099840e6}
DECODE_SOURCES = ("common.cuh", "decode.cuh")


def decode_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "decode_attention_rotate_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def decode_traffic():
    """Measured DRAM bytes per decode launch, or None once the kernel sources changed."""
    if DECODE_TRAFFIC["sources_sha256"] and DECODE_TRAFFIC["sources_sha256"] == decode_sources_sha256():
        return DECODE_TRAFFIC["bytes_per_launch"]
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        # select the GPU by UUID: CUDA_VISIBLE_DEVICES may renumber devices
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device)
        self.proc, self.lines, self.err = None, [], ""

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        try:
            self.err = self.proc.stderr.read()[-300:]
        except Exception:
            pass
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        med = float(np.median(sm)) if sm else None
        out = {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}
        if not sm:
            out["error"] = (self.err or "no samples").strip()
        return out


# ------------------------------------------------------------------ workload -------

class DecodeLayer:
    def __init__(self, w, layer, dev):
        self.tau, self.gain = W.layer_constants(w, layer)
        self.params = R.layer_params_init(self.tau, self.gain)
        Rm = torch.as_tensor(W.rotation(w.seed + layer)).to(dev)
        self.R_split = R.prepare_rotation(Rm)
        pt = torch.as_tensor(W.page_table(w))
        self.cache = R.PagedCache(int(pt.max()) + 1, pt, w.n_sink, w.n_recent, device=dev)
        self.q_c = (torch.randn((w.batch, w.heads, W.D_C), device=dev, generator=_gen(w, layer, 7))
                    .to(torch.bfloat16))
        self.q_r = (torch.randn((w.batch, w.heads, W.D_R), device=dev, generator=_gen(w, layer, 8))
                    .to(torch.bfloat16))
        self.out = torch.empty((w.batch, w.heads, W.D_C), dtype=torch.float32, device=dev)
        self.lse = torch.empty((w.batch, w.heads), dtype=torch.float32, device=dev)

    def fill(self, w, layer, dev, chunk=1 << 18):
        lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=dev)   # lengths after the fill
        for b, L in enumerate(w.seq_lens):
            for s in range(0, L, chunk):
                n = min(chunk, L - s)
                c = W.latent_device(w, layer, n, dev, stream=1000 + 97 * b + s // chunk)
                kr = W.rope_key_device(w, layer, n, dev, stream=5000 + 97 * b + s // chunk)
                req = torch.full((n,), b, dtype=torch.int32, device=dev)
                pos = torch.arange(s, s + n, dtype=torch.int32, device=dev)
                R.quantize_append(self.cache, self.params, self.R_split, c, kr, req, pos, lens)


def _gen(w, layer, k):
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed * 7919 + layer * 131 + k)
    return g


def build_decode_workload(w, dev):
    layers = [DecodeLayer(w, l, dev) for l in range(w.layers)]
    for l, lay in enumerate(layers):
        lay.fill(w, l, dev)
    torch.cuda.synchronize()
    return layers


def cache_bytes_per_step(w):
    return w.layers * w.total_tokens * R.TOKEN_BYTES


# ----------------------------------------------------------------- CPU oracle -------

def cpu_oracle_decode_rate(w, layers, budget_s=12.0):
    """The fp64 oracle decoding whole requests of the bench's layers (bounded sample)."""
    from oracle import rolaq_oracle as O
    pt = W.page_table(w)
    done_bytes, t_total, n_req = 0, 0.0, 0
    threads = torch.get_num_threads()
    for l, lay in enumerate(layers):
        pool = lay.cache.pages.cpu().numpy()
        qc = lay.q_c.float().cpu().numpy().astype(np.float64)
        qr = lay.q_r.float().cpu().numpy().astype(np.float64)
        for b, L in enumerate(w.seq_lens):
            packed, meta, kr = O.pages_read_fast(pool, pt, b, L)
            t0 = time.perf_counter()
            O.decode_request(qc[b], qr[b], packed, meta, O.bf16_bits_to_f64(kr), lay.tau, SM_SCALE)
            t_total += time.perf_counter() - t0
            done_bytes += L * R.TOKEN_BYTES
            n_req += 1
            if t_total >= budget_s:
                break
        if t_total >= budget_s:
            break
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle decode of {n_req} whole request(s) x {w.seq_lens[0]} tokens "
                      f"(16 heads, one layer each), {t_total:.1f} s"}


# ------------------------------------------------------------------ our arm --------

def pack_offsets(specs):
    """Byte layout of several tensors (shape, dtype) in one buffer, every segment 256-byte
    aligned: ([(offset, shape, dtype, nbytes)], total bytes)."""
    offs, off = [], 0
    for shape, dt in specs:
        n = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
        offs.append((off, tuple(shape), dt, n))
        off += (n + 255) // 256 * 256
    return offs, off


def pack_views(buf, offs):
    """Typed views of a uint8 buffer laid out by pack_offsets."""
    return [buf[o:o + n].view(dt).view(shape) for o, shape, dt, n in offs]


def run_ours(args, rank, world, dev):
    w = W.DECODE_4x256K_27L
    layers = build_decode_workload(w, dev)
    ws = torch.empty(R.decode_append_workspace_bytes(w.batch, w.heads), dtype=torch.uint8, device=dev)
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=dev)
    # the token appended each step overwrites the last position, so every step decodes
    # the same 262,144 tokens per request; the append runs inside the decode call (the
    # split kernel rotates the new tokens, the merge kernel stores them and adds their term)
    new_c = [W.latent_device(w, l, w.batch, dev, stream=9000) for l in range(w.layers)]
    new_kr = [W.rope_key_device(w, l, w.batch, dev, stream=9001) for l in range(w.layers)]
    stream = torch.cuda.current_stream()

    def step():
        for lay, c, kr in zip(layers, new_c, new_kr):
            R.decode_attn_append(lay.cache, lay.params, lay.R_split, c, kr, lay.q_c, lay.q_r, lens,
                                 SM_SCALE, lay.out, lay.lse, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert R.get_status() == 0

    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    ms_per_step = total_ms / args.steps
    # the step is exactly w.layers fused calls on one stream: the call's average duration
    # over the timed region (no events between the calls, which would break the overlap
    # of each call's launch with the previous one's end)
    dec_ms = ms_per_step / w.layers
    step_bytes = cache_bytes_per_step(w)
    value = aggregate_rate(step_bytes, world, ms_per_step)

    # end-to-end through the C ABI with host buffers: the step's new tokens and queries come
    # from pinned host memory (one packed buffer, one copy per step), the readouts of all
    # layers go back to pinned host memory (one packed buffer, one copy per step)
    in_src = [t for l in range(w.layers) for t in (new_c[l], new_kr[l], layers[l].q_c, layers[l].q_r)]
    in_offs, in_bytes = pack_offsets([(tuple(t.shape), t.dtype) for t in in_src])
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for hv, t in zip(pack_views(host_in, in_offs), in_src):
        hv.copy_(t.cpu())
    dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
    din = pack_views(dev_in, in_offs)
    out_specs = [spec for l in range(w.layers)
                 for spec in ((tuple(layers[l].out.shape), torch.float32), (tuple(layers[l].lse.shape), torch.float32))]
    out_offs, out_bytes = pack_offsets(out_specs)
    dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
    dout = pack_views(dev_out, out_offs)
    host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()

    def e2e_step():
        dev_in.copy_(host_in, non_blocking=True)
        for l, lay in enumerate(layers):
            c, kr, qc, qr = din[4 * l:4 * l + 4]
            R.decode_attn_append(lay.cache, lay.params, lay.R_split, c, kr, qc, qr, lens, SM_SCALE, dout[2 * l],
                                 dout[2 * l + 1], ws)
        host_out.copy_(dev_out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world) / args.steps
    h2d = host_in.numel()
    d2h = host_out.numel()
    e2e_value = aggregate_rate(step_bytes, world, e2e_ms)

    # prefill write path: 65,536 tokens x 27 layers
    q_stats = bench_quantize(args, dev, world)
    # the comparison points and the other workloads are reported beside the headline;
    # a failure in one of them is recorded in its place instead of losing the line
    bf16_stats = _guarded(bench_bf16_baseline, args, dev, world, w, dec_ms)
    bf16_stats["ours_all_protected"] = bench_all_protected(args, dev, dec_ms)
    cfg_stats = _guarded(bench_configs, args, dev)
    sweep_stats = _guarded(bench_tau_sweep, dev)
    proj_stats = [_guarded(bench_projections, args, dev, world, w.batch, w.heads),
                  _guarded(bench_projections, args, dev, world, W.PAGED_H128.batch, W.PAGED_H128.heads)]
    clocks = sampler.stop()     # sampled across the timed regions

    hbm, bf16, src = peaks()
    # the cache, plus what the fused append must read and write once per call: the rotation
    # planes, the new tokens' latents and RoPE keys, and their records
    dec_bytes = w.total_tokens * R.TOKEN_BYTES + R.RSPLIT_BYTES + w.batch * (1024 + 128 + R.TOKEN_BYTES)
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16+bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seq_lens[0], "heads": w.heads,
                   "layers": w.layers, "cache_bytes_per_step": step_bytes,
                   "l2": "inputs larger than L2 (8.15 GB cache per step), no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": decode_traffic(),
                     "kernel": "fused append + decode call (split + merge launches; duration = timed step / layers); traffic: split kernel",
                     "peak_source": src,
                     "bytes_per_launch": dec_bytes, "ms_per_launch": round(dec_ms, 4),
                     "frac_of_8tbs": round(achieved / 8000.0, 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": args.steps * w.layers * 2,
        "quantize": q_stats,
        "bf16_baseline": bf16_stats,
        "projections": proj_stats,
        "tau_sweep": sweep_stats,
        "other_workloads": cfg_stats,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_decode_rate(w, layers)
    return result


def bench_quantize(args, dev, world):
    w = W.PREFILL_64K_27L
    n = w.total_tokens
    hbm, bf16, src = peaks()
    lays = []
    for l in range(w.layers):
        tau, gain = W.layer_constants(w, l)
        pt = torch.as_tensor(W.page_table(w))
        cache = R.PagedCache(int(pt.max()) + 1, pt, device=dev)
        Rs = R.prepare_rotation(torch.as_tensor(W.rotation(w.seed + l)).to(dev))
        c = W.latent_device(w, l, n, dev)
        kr = W.rope_key_device(w, l, n, dev)
        lays.append((cache, R.layer_params_init(tau, gain), Rs, c, kr))
    req = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        for cache, p, Rs, c, kr in lays:
            R.quantize_append(cache, p, Rs, c, kr, req, pos)

    for _ in range(max(args.warmup, 1)):
        step()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world) / args.steps
    tokens = n * w.layers
    per_launch_ms = ms / w.layers
    flops = 2.0 * n * 512 * 512                     # algorithmic (one bf16-exact GEMM)
    bytes_ = n * (1024 + 128 + 288)
    return {"workload": w.name, "tokens_per_s": round(tokens * world / (ms * 1e-3), 1),
            "ms_per_step": round(ms, 4), "ms_per_launch": round(per_launch_ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(flops / (per_launch_ms * 1e-3) / 1e12, 1),
                         "peak": bf16, "unit": "TFLOP/s",
                         "frac": round(flops / (per_launch_ms * 1e-3) / 1e12 / bf16, 4),
                         "executed_flops_factor": 3, "peak_source": src},
            "hbm": {"achieved": round(bytes_ / (per_launch_ms * 1e-3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(bytes_ / (per_launch_ms * 1e-3) / 1e9 / hbm, 4)}}


# ------------------------------------------------------------ threshold sweep ----
# The write path at several thresholds tau, each with its coupled gain g(tau) from the
# library: every token of one 8,192-token request is also kept as a protected bf16 copy,
# so the stored codes, the stored statistics and bf16(y) all come from the same call.
# Reported per tau: the outer-code fraction (and 2(1 - Phi(tau)) for a normal
# coordinate), the fraction of codes that differ from those at the Lloyd-Max threshold,
# and the reconstruction response sum((x - mean)(y - mean)) / sum((y - mean)^2) with the
# coupled gain (unit response is the aim) and at gain 1, plus the normalised error.
SWEEP_TAUS = (0.85, 0.88, 0.91, 0.94, 0.9816, 1.02, 1.06, 1.10)
LLOYD_MAX_TAU = 0.9816


def unpack_codes(pages, n):
    """Codes [n, 512] of a request laid out on consecutive pages (byte b of a token holds
    coordinates 4b..4b+3, coordinate j at bits 2(j % 4))."""
    pg = pages.reshape(-1, R.PAGE_BYTES)[:, :R.PAGE_TOKENS * R.CODE_BYTES]
    b = pg.reshape(-1, R.CODE_BYTES)[:n].astype(np.uint8)
    return np.stack([(b >> (2 * j)) & 3 for j in range(4)], axis=2).reshape(n, R.D_C)


def unpack_meta(pages, n):
    off = R.PAGE_TOKENS * R.CODE_BYTES
    pg = pages.reshape(-1, R.PAGE_BYTES)[:, off:off + R.PAGE_TOKENS * R.META_BYTES]
    return np.ascontiguousarray(pg).view(np.float32).reshape(-1, R.GROUPS, 2)[:n].astype(np.float64)


def bench_tau_sweep(dev, n=8192):
    w = W.Workload("tau_sweep_8k", 1, (n,), 16, n_sink=n, seed=4250)
    pt = torch.as_tensor(W.page_table(w))
    Rs = R.prepare_rotation(torch.as_tensor(W.rotation(w.seed)).to(dev))
    c = W.latent_device(w, 0, n, dev)
    kr = W.rope_key_device(w, 0, n, dev)
    req = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    rows, ref = [], None
    runs = {}
    for tau in SWEEP_TAUS:
        gain, kappa1 = R.coupled_gain(tau)
        p = R.layer_params_init(tau, gain)
        cache = R.PagedCache(int(pt.max()) + 1, pt, n_sink=n, device=dev)
        R.quantize_append(cache, p, Rs, c, kr, req, pos)
        torch.cuda.synchronize()
        pages = cache.pages.cpu().numpy()
        y = cache.prot[0].float().cpu().numpy().astype(np.float64).reshape(n, R.GROUPS, R.GROUP)
        runs[tau] = (unpack_codes(pages, n), unpack_meta(pages, n), y, p, gain, kappa1)
    ref = runs[LLOYD_MAX_TAU][0]
    for tau in SWEEP_TAUS:
        codes, meta, y, p, gain, kappa1 = runs[tau]
        lev = np.array([-p.level_b, -p.level_a, p.level_a, p.level_b], dtype=np.float64)
        mu, scale = meta[:, :, 0:1], meta[:, :, 1:2]
        xc = scale * lev[codes.reshape(n, R.GROUPS, R.GROUP)]        # x - mean, coupled gain
        yc = y - mu
        den = float((yc * yc).sum())
        resp = float((xc * yc).sum()) / den
        rows.append({"tau": tau, "gain": round(gain, 6), "kappa_gain1": round(kappa1, 6),
                     "outer_code_frac": round(float(np.isin(codes, (0, 3)).mean()), 5),
                     "outer_frac_normal": round(1.0 - math.erf(tau / math.sqrt(2.0)), 5),
                     "code_flip_frac_vs_lloyd_max": round(float((codes != ref).mean()), 5),
                     "response": round(resp, 5), "response_gain1": round(resp / gain, 5),
                     "nmse": round(float(((xc - yc) ** 2).sum()) / den, 5),
                     "nmse_gain1": round(float(((xc / gain - yc) ** 2).sum()) / den, 5)})
    return {"workload": w.name, "tokens": n, "lloyd_max_tau": LLOYD_MAX_TAU,
            "y_source": "bf16 side-store copy written by the same call", "rows": rows}


def capture_graph(fn):
    """Record fn's launches (on a side stream, after one eager warm-up call) into a CUDA graph."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


# ------------------------------------------------------- the other workloads ----
# Decode on the other decode workloads, each over enough layers that one sweep of
# the caches exceeds L2 (126 MB): 4 x 32K at 16 heads, 32 requests of log-uniform lengths
# at 128 heads on shuffled pages, and 64 x 8K with 4 sink + 128 recent bf16 tokens.

def algorithmic_decode_bytes(w):
    """2-bit tokens at 288 B, protected tokens at 1,152 B (bf16 latent + RoPE key)."""
    total = 0
    for L in w.seq_lens:
        prot = min(L, w.n_sink + w.n_recent) if (w.n_sink or w.n_recent) else 0
        total += (L - prot) * R.TOKEN_BYTES + prot * R.BF16_TOKEN_BYTES
    return total


def bench_configs(args, dev):
    hbm, bf16, src = peaks()
    res = []
    for w in (W.DECODE_4x32K, W.PAGED_H128, W.MIXED_64x8K):
        per_layer = algorithmic_decode_bytes(w)
        nl = max(2, -(-300_000_000 // per_layer))
        layers = []
        for l in range(nl):
            lay = DecodeLayer(w, l, dev)
            lay.fill(w, l, dev)
            layers.append(lay)
        ws = torch.empty(R.decode_workspace_bytes(w.batch, w.heads), dtype=torch.uint8, device=dev)
        lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=dev)

        def sweep():
            for lay in layers:
                R.decode_attn(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE, lay.out, lay.lse, ws)

        for _ in range(max(args.warmup, 3)):
            sweep()
        torch.cuda.synchronize()
        assert R.get_status() == 0
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        t0.record()
        for _ in range(reps):
            sweep()
        t1.record()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / (reps * nl)
        gbs = per_layer / (ms * 1e-3) / 1e9
        entry = {"workload": w.name, "batch": w.batch, "heads": w.heads, "tokens": w.total_tokens,
                 "n_sink": w.n_sink, "n_recent": w.n_recent, "layers_swept": nl,
                 "bytes_per_layer": per_layer, "ms_per_layer": round(ms, 4),
                 "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                              "frac": round(gbs / hbm, 4), "frac_of_8tbs": round(gbs / 8000.0, 4),
                              "peak_source": src}}
        if w.heads >= 128:
            flops = 2.0 * w.heads * (R.D_C + R.D_R + R.D_C) * w.total_tokens
            tf = flops / (ms * 1e-3) / 1e12
            entry["tensor"] = {"achieved": round(tf, 1), "peak": bf16, "unit": "TFLOP/s",
                               "frac": round(tf / bf16, 4), "flops_per_layer": flops}
        res.append(entry)
        del layers, ws
        torch.cuda.empty_cache()
    return res


# ------------------------------------------------------ absorbed projections ----
# Per decode step and layer: the query fold before the cache read and the output unfold
# after it, over one set of folded bf16 weights per layer; enough layers that the weights
# of one sweep exceed L2 (every call reads its weights from HBM).

def bench_projections(args, dev, world, batch, heads):
    per_layer = 2 * heads * R.D_NOPE * R.D_C * 2                   # W_q + W_o, bf16
    layers = max(27, -(-300_000_000 // per_layer))                 # > 2 x the 126 MB L2
    g = W.device_generator(4242 + heads, dev)
    Wq = [(torch.randn((heads, R.D_NOPE, R.D_C), generator=g, device=dev) / 11.3).to(torch.bfloat16)
          for _ in range(layers)]
    Wo = [(torch.randn((heads, R.D_C, R.D_V), generator=g, device=dev) / 22.6).to(torch.bfloat16)
          for _ in range(layers)]
    q = torch.randn((batch, heads, R.D_NOPE), generator=g, device=dev).to(torch.bfloat16)
    o = torch.randn((batch, heads, R.D_C), generator=g, device=dev)
    qc = torch.empty((batch, heads, R.D_C), dtype=torch.bfloat16, device=dev)
    v = torch.empty((batch, heads, R.D_V), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def calls():
        for l in range(layers):
            R.fold_query(q, Wq[l], out=qc)
            R.unfold_output(o, Wo[l], v=v)

    graph = capture_graph(calls)          # launches only: the host's per-call cost stays out
    sweep = graph.replay
    for _ in range(max(args.warmup, 3)):
        sweep()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    reps = 5
    t0.record(stream)
    for _ in range(reps):
        sweep()
    t1.record(stream)
    torch.cuda.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / (reps * layers)               # one fold + one unfold
    bytes_ = per_layer + batch * heads * (R.D_NOPE * 2 + R.D_C * 2 + R.D_C * 4 + R.D_V * 4)
    hbm, _, src = peaks()
    gbs = bytes_ / (us * 1e-6) / 1e9
    return {"batch": batch, "heads": heads, "us_per_layer": round(us, 3), "bytes_per_layer": bytes_,
            "layers_swept": layers, "launches_per_layer": 2, "timing": "CUDA graph of one sweep",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src}}


# ------------------------------------------------------------- BF16 baseline ----
# The same decode on an uncompressed cache (1,152 B per token: 512 bf16 latent + 64 bf16
# RoPE key, 64-token pages), run by a library kernel: FlashInfer's TRT-LLM-generated MLA
# decode for Blackwell.  It is a comparison point (the pages compare their 2-bit decode
# with BF16 on the same GPU), never part of this library's path.

def bench_bf16_baseline(args, dev, world, w, dec_ms):
    try:
        from flashinfer import mla as fi_mla
    except Exception as e:                      # library missing: no baseline, say why
        return {"unavailable": f"flashinfer not importable: {type(e).__name__}"}
    B, L, H = w.batch, w.seq_lens[0], w.heads
    page = R.PAGE_TOKENS
    npg = (L + page - 1) // page
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    kv = torch.randn((B * npg, page, 576), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    bt = torch.arange(B * npg, dtype=torch.int32, device=dev).reshape(B, npg)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    q = torch.randn((B, 1, H, 576), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    ws = torch.zeros(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        fi_mla.trtllm_batch_decode_with_kv_cache_mla(q, kv, ws, 128, 512, 64, bt, lens, L,
                                                    bmm1_scale=SM_SCALE, bmm2_scale=1.0)

    for _ in range(max(args.warmup, 1)):
        call()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    reps = max(args.steps, 1) * 4
    t0.record(stream)
    for _ in range(reps):
        call()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world) / reps
    nbytes = B * L * 1152
    del kv
    return {"kernel": "flashinfer trtllm_batch_decode_with_kv_cache_mla (library), bf16 cache",
            "workload": f"{B} x {L} tokens, {H} heads, one layer", "bytes_per_token": 1152,
            "ms_per_call": round(ms, 4), "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "tokens_per_s": round(B * L / (ms * 1e-3), 1),
            "time_ratio_bf16_over_2bit": round(ms / dec_ms, 3), "capacity_ratio": 4.0}


def bench_all_protected(args, dev, dec_ms):
    """This library's decode with quantization disabled: every token protected, its bf16
    latent read from the side store (1,152 B per token with the RoPE key), the same
    4 x 262,144 tokens at 16 heads as the bench; through the BF16 decode
    (rolaq_decode_attn_bf16), and for comparison through the 2-bit-page decode, which
    still stages each token's page."""
    w = W.Workload("all_protected_4x256k_h16", 4, (262144,) * 4, 16, n_sink=0, n_recent=262144, seed=1010)
    hbm, _, src = peaks()
    try:
        lay = DecodeLayer(w, 0, dev)
        lay.fill(w, 0, dev)
        ws = torch.empty(R.decode_workspace_bytes(w.batch, w.heads), dtype=torch.uint8, device=dev)
        lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=dev)

        def timed(fn):
            for _ in range(max(args.warmup, 3)):
                fn()
            torch.cuda.synchronize()
            assert R.get_status() == 0
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 10
            t0.record()
            for _ in range(reps):
                fn()
            t1.record()
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / reps
        ms = timed(lambda: R.decode_attn_bf16(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE, lay.out,
                                              lay.lse, ws))
        ms2 = timed(lambda: R.decode_attn(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE, lay.out,
                                          lay.lse, ws))
    except Exception as e:                      # report, never lose the bench line
        return {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    finally:
        torch.cuda.empty_cache()
    nbytes = w.total_tokens * R.BF16_TOKEN_BYTES
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "rolaq_decode_bf16 + merge (BF16 decode: side-store rows and RoPE rows by bulk tensor copies)",
            "workload": "4 x 262144 tokens, 16 heads, one layer", "bytes_per_token": R.BF16_TOKEN_BYTES,
            "ms_per_call": round(ms, 4), "GB_s": round(gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src},
            "time_ratio_over_2bit": round(ms / dec_ms, 3),
            "via_2bit_page_decode": {"ms_per_call": round(ms2, 4),
                                     "GB_s": round(nbytes / (ms2 * 1e-3) / 1e9, 1)}}


# ------------------------------------------------------------ profiling cases ----
# Small single-kernel cases for ncu captures (inputs larger than L2, a few hundred MB on
# the device): `--case decode` runs one layer of 4 requests x 131,072 tokens at 16 heads,
# `--case quantize` the write path on 262,144 tokens, `--case project` the query fold and
# output unfold for 32 requests x 128 heads.  They print their own timing.

def run_case(args, dev):
    if args.case == "protected":
        print(json.dumps({"case": "protected", "result": bench_all_protected(args, dev, float("nan"))}), flush=True)
        return
    if args.case == "sweep":
        print(json.dumps({"case": "sweep", "result": bench_tau_sweep(dev)}), flush=True)
        return
    if args.case == "configs":
        print(json.dumps({"case": "configs", "results": bench_configs(args, dev)}), flush=True)
        return
    if args.case == "decode":
        w = W.Workload("decode_4x128k_h16", 4, (131072,) * 4, 16, seed=4242)
        lay = DecodeLayer(w, 0, dev)
        lay.fill(w, 0, dev)
        ws = torch.empty(R.decode_workspace_bytes(w.batch, w.heads), dtype=torch.uint8, device=dev)
        lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=dev)
        fn = lambda: R.decode_attn(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE, lay.out, lay.lse, ws)
        nbytes = w.total_tokens * R.TOKEN_BYTES
    elif args.case == "project":
        # query fold + output unfold, 32 requests x 128 heads, ten layers' weights in turn
        B, H, nl = 32, 128, 10
        g = W.device_generator(4244, dev)
        Wq = [(torch.randn((H, R.D_NOPE, R.D_C), generator=g, device=dev) / 11.3).to(torch.bfloat16)
              for _ in range(nl)]
        Wo = [(torch.randn((H, R.D_C, R.D_V), generator=g, device=dev) / 22.6).to(torch.bfloat16)
              for _ in range(nl)]
        q = torch.randn((B, H, R.D_NOPE), generator=g, device=dev).to(torch.bfloat16)
        o = torch.randn((B, H, R.D_C), generator=g, device=dev)
        qc = torch.empty((B, H, R.D_C), dtype=torch.bfloat16, device=dev)
        v = torch.empty((B, H, R.D_V), dtype=torch.float32, device=dev)
        # the ten layers' calls in one CUDA graph: the host's per-call cost stays out of the timing
        graph = capture_graph(lambda: [(R.fold_query(q, Wq[l], out=qc), R.unfold_output(o, Wo[l], v=v))
                                       for l in range(nl)])
        fn = graph.replay
        w = W.Workload("project_b32_h128", B, (1,) * B, H, seed=4244)
        nbytes = nl * (2 * H * R.D_NOPE * R.D_C * 2 + B * H * (R.D_NOPE * 2 + R.D_C * 2 + R.D_C * 4 + R.D_V * 4))
    else:
        w = W.Workload("quantize_262k", 1, (262144,), 16, seed=4243)
        n = w.total_tokens
        tau, gain = W.layer_constants(w, 0)
        pt = torch.as_tensor(W.page_table(w))
        cache = R.PagedCache(int(pt.max()) + 1, pt, device=dev)
        Rs = R.prepare_rotation(torch.as_tensor(W.rotation(w.seed)).to(dev))
        p = R.layer_params_init(tau, gain)
        c = W.latent_device(w, 0, n, dev)
        kr = W.rope_key_device(w, 0, n, dev)
        req = torch.zeros(n, dtype=torch.int32, device=dev)
        pos = torch.arange(n, dtype=torch.int32, device=dev)
        fn = lambda: R.quantize_append(cache, p, Rs, c, kr, req, pos)
        nbytes = n * (1024 + 128 + 288)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"case": args.case, "workload": w.name, "ms_per_call": round(ms, 4),
                      "algorithmic_GBps": round(nbytes / ms / 1e6, 1), "status": R.get_status()}), flush=True)


# ---------------------------------------------------------------- reference arm ----

def run_reference(args, rank, world):
    """The CPU oracle on this arm's workload: each step decodes one whole request of one
    layer (262,144 tokens, fp64) on the host cores."""
    from oracle import rolaq_oracle as O
    w = W.DECODE_4x256K_27L
    L = w.seq_lens[0]
    rng = np.random.default_rng(w.seed)
    tau, gain = W.layer_constants(w, 0)
    packed = rng.integers(0, 256, size=(L, 128), dtype=np.uint8)
    meta = np.stack([rng.standard_normal((L, 4)), np.abs(rng.standard_normal((L, 4))) + 0.5],
                    axis=2).astype(np.float32)
    kr = rng.standard_normal((L, 64))
    qc = rng.standard_normal((w.heads, 512))
    qr = rng.standard_normal((w.heads, 64))

    def step():
        O.decode_request(qc, qr, packed, meta, kr, tau, SM_SCALE)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = L * R.TOKEN_BYTES / dt / 1e9
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": L, "heads": w.heads,
                       "layers": w.layers},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": torch.get_num_threads(),
                             "kind": "oracle",
                             "sample": f"each step: one request x {L} tokens of one layer, fp64 oracle"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------- plumbing -------

def _guarded(fn, *a):
    try:
        return fn(*a)
    except Exception as e:
        return {"unavailable": f"{type(e).__name__}: {e}"[:200]}


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The slowest rank's time: every rank passes its own, all get the maximum."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(bytes_per_rank_step, world, ms_per_step):
    """Whole-job throughput in GB/s: every rank processes its own replica of the workload
    (weak scaling), timed by the slowest rank."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["decode", "quantize", "project", "configs", "protected", "sweep"], default=None,
                    help="run one small single-kernel case (for ncu captures) instead of the bench")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 1)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    R.lib()
    if args.case:
        run_case(args, dev)
        return
    res = run_ours(args, rank, world, dev)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
