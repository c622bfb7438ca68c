"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import (DECODE_TOL, META_TOL, SM_SCALE, bf16_bits, build_oracle_cache,
                               codes_match, f64, meta_match, oracle_decode, rel_l2)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    R.lib()
    yield
    assert R.get_status() == 0


def _quantize_on_gpu(w, layer, seq_lens, tau, gain, n_sink=0, n_recent=0, zero_latent=False):
    Rm = W.rotation(w.seed + layer)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(W.Workload(w.name, len(seq_lens), tuple(seq_lens), w.heads,
                                 paged_shuffled=w.paged_shuffled, seed=w.seed))
    num_pages = int(pt.max() + 1)
    cache = R.PagedCache(num_pages, torch.as_tensor(pt), n_sink, n_recent, device=DEV)
    cache.pages.fill_(0xAB)                       # unwritten bytes must stay untouched
    cs, krs, reqs, poss = [], [], [], []
    for r, L in enumerate(seq_lens):
        c = W.latent(w, layer, L, stream=100 + r)
        if zero_latent:
            c = torch.zeros_like(c)
        cs.append(c)
        krs.append(W.rope_key(w, layer, L, stream=200 + r))
        reqs.append(torch.full((L,), r, dtype=torch.int32))
        poss.append(torch.arange(L, dtype=torch.int32))
    c = torch.cat(cs).to(DEV)
    kr = torch.cat(krs).to(DEV)
    req = torch.cat(reqs).to(DEV)
    pos = torch.cat(poss).to(DEV)
    lens = torch.as_tensor(seq_lens, dtype=torch.int32).to(DEV)
    p = R.layer_params_init(tau, gain)
    R.quantize_append(cache, p, R_split, c, kr, req, pos, lens)
    torch.cuda.synchronize()
    return cache, cs, krs, Rm.astype(np.float64), pt


def _check_write(cache, cs, krs, Rm, pt, seq_lens, tau, gain, n_sink=0, n_recent=0):
    pool = cache.pages.cpu().numpy()
    frac_total, n_total = 0.0, 0
    prot = cache.prot.float().cpu().numpy() if cache.prot is not None else None
    for r, L in enumerate(seq_lens):
        if L == 0:
            continue
        q = O.quantize(f64(cs[r]), Rm, tau, gain)
        packed, meta, kr = O.pages_read_fast(pool, pt, r, L)
        ok, frac, nbad = codes_match(packed, q, tau)
        assert ok, f"request {r}: {nbad} codes differ outside the threshold window"
        frac_total += frac * L
        n_total += L
        emu, es = meta_match(meta, q, gain)
        assert emu <= META_TOL and es <= META_TOL, (emu, es)
        assert (kr == bf16_bits(krs[r])).all()
        if prot is not None:
            yb = O.bf16_round(q["y"])
            for p in range(L):
                if p < n_sink:
                    slot = p
                elif p >= L - n_recent:
                    slot = n_sink + p % n_recent
                else:
                    continue
                # bf16 of an fp32 y whose error is ~1e-6 of the token's magnitude: one bf16
                # ulp apart, plus that error for coordinates near zero
                d = np.abs(prot[r, slot] - yb[p])
                tol = np.abs(yb[p]) * 2.0 ** -7 + 1e-5 * np.abs(q["y"][p]).max()
                assert (d <= tol).all(), (p, float((d - tol).max()))
    return frac_total / max(n_total, 1)


def test_quantize_tiny():
    w = W.TINY
    frac = None
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, [256], 0.9816, 1.16)
    frac = _check_write(cache, cs, krs, Rm, pt, [256], 0.9816, 1.16)
    assert frac < 1e-3


def test_quantize_ragged_multi_request_shuffled_pages():
    w = W.Workload("ragged", 3, (1, 300, 129), 16, paged_shuffled=True, seed=77)
    tau, gain = 0.87, 1.07
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, [1, 300, 129], tau, gain)
    _check_write(cache, cs, krs, Rm, pt, [1, 300, 129], tau, gain)
    # bytes of pages no token was written to are untouched
    pool = cache.pages.cpu().numpy().reshape(-1, O.PAGE_BYTES)
    assert (pool[pt[0, 0], 288 * 0 + 128:O.PAGE_META] == 0xAB).all()


@pytest.mark.parametrize("n", [1, 5, 8, 13, 64])
def test_small_append_token_counts(n):
    """Calls of up to 64 tokens take the clustered small-append kernel: blocks of 8 tokens
    with a ragged last block, scattered positions of several requests, sink and recent
    positions included; every record against the oracle, other rows untouched."""
    B, cap, n_sink, n_recent = 4, 256, 4, 16
    w = W.Workload(f"sa{n}", B, (cap,) * B, 16, paged_shuffled=True, seed=500 + n)
    tau, gain = 0.93, 1.09
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    cache = R.PagedCache(int(pt.max()) + 1, torch.as_tensor(pt), n_sink, n_recent, device=DEV)
    cache.pages.fill_(0xAB)
    rng = np.random.default_rng(n)
    flat = rng.choice(B * cap, n, replace=False)
    flat[0] = 2                                    # a sink position
    if n > 1:
        flat[1] = cap + cap - 1                    # a recent position of request 1
    flat = np.unique(flat)
    rng.shuffle(flat)
    req = (flat // cap).astype(np.int32)
    pos = (flat % cap).astype(np.int32)
    m = len(flat)
    c = W.latent(w, 0, m, stream=7)
    kr = W.rope_key(w, 0, m, stream=8)
    lens = torch.full((B,), cap, dtype=torch.int32, device=DEV)
    p = R.layer_params_init(tau, gain)
    R.quantize_append(cache, p, R_split, c.to(DEV), kr.to(DEV), torch.as_tensor(req).to(DEV),
                      torch.as_tensor(pos).to(DEV), lens)
    torch.cuda.synchronize()
    pool = cache.pages.cpu().numpy()
    q = O.quantize(f64(c), Rm.astype(np.float64), tau, gain)
    recs = [O.pages_read(pool, pt, int(b), int(s) + 1, start=int(s)) for b, s in zip(req, pos)]
    packed = np.stack([x[0][0] for x in recs])
    meta = np.stack([x[1][0] for x in recs])
    krb = np.stack([x[2][0] for x in recs])
    ok, frac, nbad = codes_match(packed, q, tau)
    assert ok, nbad
    emu, es = meta_match(meta, q, gain)
    assert emu <= META_TOL and es <= META_TOL, (emu, es)
    assert (krb == bf16_bits(kr)).all()
    prot = cache.prot.float().cpu().numpy().astype(np.float64)
    seen = 0
    for t, (b, s) in enumerate(zip(req, pos)):
        if s < n_sink:
            slot = s
        elif s >= cap - n_recent:
            slot = n_sink + s % n_recent
        else:
            continue
        seen += 1
        y = q["y"][t]
        tol = np.abs(y) * 2.0 ** -7 + 1e-5 * np.abs(y).max()
        assert (np.abs(prot[b, slot] - y) <= tol).all(), (b, s)
    assert seen >= 1
    pages = pool.reshape(-1, O.PAGE_BYTES)
    written = set(zip(req.tolist(), pos.tolist()))
    for b in range(B):
        for s in range(0, cap, 7):
            if (b, s) not in written:
                row = s % O.PAGE_TOKENS
                assert (pages[pt[b, s // O.PAGE_TOKENS], row * 128:(row + 1) * 128] == 0xAB).all(), (b, s)


def test_quantize_protected_side_store():
    w = W.Workload("prot", 2, (200, 40), 16, seed=78)
    tau, gain = 1.05, 1.12
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, [200, 40], tau, gain, n_sink=4, n_recent=16)
    _check_write(cache, cs, krs, Rm, pt, [200, 40], tau, gain, 4, 16)


def test_quantize_zero_latent_group():
    w = W.Workload("zero", 1, (70,), 16, seed=79)
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, [70], 0.95, 1.1, zero_latent=True)
    packed, meta, _ = O.pages_read_fast(cache.pages.cpu().numpy(), pt, 0, 70)
    assert (O.unpack(packed) == 2).all()
    assert (meta == 0).all()


def _decode_case(w, seq_lens, H, tau, gain, n_sink=0, n_recent=0, layer=0):
    cache, data, Rm = build_oracle_cache(w, layer, seq_lens, tau, gain, n_sink, n_recent)
    B = len(seq_lens)
    ww = W.Workload(w.name, B, tuple(seq_lens), H, seed=w.seed)
    q_c, q_r = W.queries(ww, layer)
    p = R.layer_params_init(tau, gain)
    lens = torch.as_tensor(seq_lens, dtype=torch.int32).to(DEV)
    out, lse = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_decode(data, f64(q_c), f64(q_r), seq_lens, tau, SM_SCALE, n_sink, n_recent)
    out = out.cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    for r, L in enumerate(seq_lens):
        if L == 0:
            assert (out[r] == 0).all() and np.isneginf(lse[r]).all()
            continue
        e = rel_l2(out[r], o_ref[r])
        assert e.max() <= DECODE_TOL, (r, e.max())
        assert np.abs(lse[r] - l_ref[r]).max() <= 1e-2 * max(1.0, np.abs(l_ref[r]).max()), r
    return out, o_ref


def test_decode_tiny():
    _decode_case(W.TINY, [256], 16, 0.9816, 1.16)


@pytest.mark.parametrize("H", [16, 32])
def test_decode_ragged_lengths_and_empty(H):
    w = W.Workload("dr", 5, (1, 63, 64, 65, 0), H, paged_shuffled=True, seed=90)
    _decode_case(w, [1, 63, 64, 65, 0], H, 0.9, 1.05)


def test_decode_plan_fits_one_wave():
    """40 requests of log-uniform lengths: the first chunk size leaves more work items
    than SMs, so the plan raises it until they fit one wave; every request must still be
    covered exactly once by its items."""
    rng = np.random.default_rng(98)
    lens = [int(x) for x in np.exp(rng.uniform(np.log(64), np.log(20000), size=40)).round()]
    w = W.Workload("wave", len(lens), tuple(lens), 16, paged_shuffled=True, seed=98)
    _decode_case(w, lens, 16, 0.92, 1.07)


def test_decode_several_splits():
    # 3 requests of a few thousand tokens: many split-K items per request
    w = W.Workload("ds", 3, (4096, 3000, 777), 16, paged_shuffled=True, seed=91)
    _decode_case(w, [4096, 3000, 777], 16, 0.93, 1.18)


def test_decode_128_heads_paged():
    w = W.Workload("h128", 4, (1024, 2500, 64, 1500), 128, paged_shuffled=True, seed=92)
    _decode_case(w, [1024, 2500, 64, 1500], 128, 0.88, 1.02)


@pytest.mark.parametrize("H", [32, 48, 64])
def test_decode_head_counts(H):
    # 32 and 64 heads take 32-head CTAs, 48 heads three 16-head CTAs per work item
    w = W.Workload("hc%d" % H, 3, (700, 64, 1999), H, paged_shuffled=True, seed=97 + H)
    _decode_case(w, [700, 64, 1999], H, 0.93, 1.08, n_sink=4, n_recent=64)


def test_decode_sink_and_recent_protection():
    w = W.Workload("mix", 3, (1000, 130, 5), 16, seed=93)
    _decode_case(w, [1000, 130, 5], 16, 0.97, 1.1, n_sink=4, n_recent=128)


def test_decode_single_token_equals_its_reconstruction():
    w = W.Workload("one", 1, (1,), 16, seed=94)
    out, ref = _decode_case(w, [1], 16, 0.9, 1.0)
    assert rel_l2(out[0], ref[0]).max() < 5e-3


def test_end_to_end_write_then_decode():
    """Cache written by the GPU write path and decoded on the GPU, against the oracle
    quantizing the same latents itself and decoding its own records."""
    w = W.Workload("e2e", 2, (700, 1333), 16, paged_shuffled=True, seed=95)
    tau, gain = 0.91, 1.13
    lens_l = [700, 1333]
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, lens_l, tau, gain, n_sink=4, n_recent=128)
    q_c, q_r = W.queries(W.Workload("e2e", 2, tuple(lens_l), 16, seed=95), 0)
    p = R.layer_params_init(tau, gain)
    lens = torch.as_tensor(lens_l, dtype=torch.int32).to(DEV)
    out, lse = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    torch.cuda.synchronize()
    _, data, _ = build_oracle_cache(w, 0, lens_l, tau, gain, n_sink=4, n_recent=128)
    o_ref, _ = oracle_decode(data, f64(q_c), f64(q_r), lens_l, tau, SM_SCALE, 4, 128)
    for r in range(len(lens_l)):
        e = rel_l2(out[r].cpu().numpy().astype(np.float64), o_ref[r])
        assert e.max() <= DECODE_TOL, e.max()


@pytest.mark.parametrize("H", [16, 32])
def test_bad_page_entry_sets_status_and_skips(H):
    w = W.Workload("bad", 1, (256,), H, seed=96)
    cache, data, _ = build_oracle_cache(w, 0, [256], 0.9, 1.0)
    cache.page_table[0, 1] = cache.num_pages + 5          # outside the pool
    q_c, q_r = W.queries(w, 0)
    p = R.layer_params_init(0.9, 1.0)
    lens = torch.tensor([256], dtype=torch.int32, device=DEV)
    out, _ = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    st = R.get_status()
    assert st & R.STATUS_BAD_PAGE
    assert torch.isfinite(out).all()
    # tokens of the skipped page are left out: compare with the oracle on the other pages
    keep = np.r_[0:64, 128:256]
    d = data[0]
    xq = O.dequantize(d["q"]["packed"], d["q"]["meta"], 0.9)[keep]
    o_ref, _ = O.attend(f64(q_c[0]), f64(q_r[0]), xq, d["k_r"][keep], SM_SCALE)
    assert rel_l2(out[0].cpu().numpy().astype(np.float64), o_ref).max() <= DECODE_TOL


def test_quantize_metadata_tail_over_a_million_groups():
    """Codes and metadata over 262,144 tokens (1,048,576 groups), the decode-shaped latent
    distribution: the worst group still meets the tolerances."""
    w = W.Workload("tail", 1, (262144,), 16, seed=97)
    tau, gain = 0.93, 1.14
    cache, cs, krs, Rm, pt = _quantize_on_gpu(w, 0, [262144], tau, gain)
    packed, meta, kr = O.pages_read_fast(cache.pages.cpu().numpy(), pt, 0, 262144)
    q = O.quantize(f64(cs[0]), Rm, tau, gain)
    ok, frac, nbad = codes_match(packed, q, tau)
    emu, es = meta_match(meta, q, gain)
    print(f"\nwrite-path tail: codes in window {frac:.2e}, mismatches outside {nbad}, "
          f"max mean err {emu:.3e}, max scale err {es:.3e}")
    assert ok, nbad
    assert emu <= META_TOL and es <= META_TOL, (emu, es)


def test_streaming_append_with_recent_ring():
    """Prefill, then one token per request per step (the small-append kernel), with 4 sink
    and 16 recent tokens protected: every record, the side store after the ring has
    wrapped, and the decode of the final cache match the oracle."""
    L0 = [100, 64, 130]
    steps = 20
    B = len(L0)
    tau, gain = 0.94, 1.09
    n_sink, n_recent = 4, 16
    w = W.Workload("stream", B, tuple(l + steps for l in L0), 16, paged_shuffled=True, seed=98)
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    cache = R.PagedCache(int(pt.max() + 1), torch.as_tensor(pt), n_sink, n_recent, device=DEV)
    p = R.layer_params_init(tau, gain)
    Lf = [l + steps for l in L0]
    lat = [W.latent(w, 0, Lf[r], stream=100 + r) for r in range(B)]
    kr = [W.rope_key(w, 0, Lf[r], stream=200 + r) for r in range(B)]
    # prefill (tensor-core path for the 294 tokens)
    c = torch.cat([lat[r][:L0[r]] for r in range(B)]).to(DEV)
    k = torch.cat([kr[r][:L0[r]] for r in range(B)]).to(DEV)
    req = torch.cat([torch.full((L0[r],), r, dtype=torch.int32) for r in range(B)]).to(DEV)
    pos = torch.cat([torch.arange(L0[r], dtype=torch.int32) for r in range(B)]).to(DEV)
    R.quantize_append(cache, p, R_split, c, k, req, pos, torch.as_tensor(L0, dtype=torch.int32).to(DEV))
    # one token per request per step
    for s in range(steps):
        c = torch.stack([lat[r][L0[r] + s] for r in range(B)]).to(DEV)
        k = torch.stack([kr[r][L0[r] + s] for r in range(B)]).to(DEV)
        req = torch.arange(B, dtype=torch.int32, device=DEV)
        pos = torch.as_tensor([L0[r] + s for r in range(B)], dtype=torch.int32).to(DEV)
        lens = torch.as_tensor([L0[r] + s + 1 for r in range(B)], dtype=torch.int32).to(DEV)
        R.quantize_append(cache, p, R_split, c, k, req, pos, lens)
    torch.cuda.synchronize()
    pool = cache.pages.cpu().numpy()
    prot = cache.prot.float().cpu().numpy().astype(np.float64)
    q_c, q_r = W.queries(w, 0)
    lens = torch.as_tensor(Lf, dtype=torch.int32).to(DEV)
    out, _ = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    out = out.cpu().numpy().astype(np.float64)
    for r in range(B):
        L = Lf[r]
        q = O.quantize(f64(lat[r]), Rm.astype(np.float64), tau, gain)
        packed, meta, krb = O.pages_read_fast(pool, pt, r, L)
        ok, frac, nbad = codes_match(packed, q, tau)
        assert ok, (r, nbad)
        emu, es = meta_match(meta, q, gain)
        assert emu <= META_TOL and es <= META_TOL, (r, emu, es)
        assert (krb == bf16_bits(kr[r])).all()
        yb = O.bf16_round(q["y"])
        content = np.zeros((L, 512))
        for pp in range(L):
            if pp < n_sink:
                slot = pp
            elif pp >= L - n_recent:
                slot = n_sink + pp % n_recent
            else:
                continue
            d = np.abs(prot[r, slot] - yb[pp])
            assert (d <= np.abs(yb[pp]) * 2.0 ** -7 + 1e-5 * np.abs(q["y"][pp]).max()).all(), (r, pp)
            content[pp] = prot[r, slot]
        o_ref, _ = O.decode_request(f64(q_c[r]), f64(q_r[r]), packed, meta, O.bf16_bits_to_f64(krb), tau,
                                    SM_SCALE, content, n_sink, n_recent)
        assert rel_l2(out[r], o_ref).max() <= DECODE_TOL


def test_decode_fp16_range_status():
    """x and the content query enter the decode MMAs as fp16: a cache whose decoded values
    pass 65504, or a query element that large, sets ROLAQ_STATUS_RANGE (the result of that
    call is not valid); an ordinary call leaves the status clean."""
    w = W.Workload("range", 1, (200,), 16, seed=97)
    tau, gain = 0.95, 1.1
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    p = R.layer_params_init(tau, gain)
    lens = torch.tensor([200], dtype=torch.int32, device=DEV)
    q_c, q_r = W.queries(w, 0)
    q_c, q_r = q_c.to(DEV), q_r.to(DEV)
    req = torch.zeros(200, dtype=torch.int32, device=DEV)
    pos = torch.arange(200, dtype=torch.int32, device=DEV)
    kr = W.rope_key(w, 0, 200).to(DEV)

    def cache_with(scale):
        cache = R.PagedCache(int(pt.max()) + 1, torch.as_tensor(pt), device=DEV)
        c = (W.latent(w, 0, 200).float() * scale).to(torch.bfloat16).to(DEV)
        R.quantize_append(cache, p, R_split, c, kr, req, pos, lens)
        return cache

    assert R.get_status() == 0
    ok = cache_with(1.0)
    R.decode_attn(ok, p, q_c, q_r, lens, SM_SCALE)
    assert R.get_status() == 0
    big = cache_with(1.0e5)
    R.decode_attn(big, p, q_c, q_r, lens, SM_SCALE)
    assert R.get_status() & R.STATUS_RANGE
    q_big = q_c.clone()
    q_big[0, 3, 17] = 1.0e5
    R.decode_attn(ok, p, q_big, q_r, lens, SM_SCALE)
    assert R.get_status() & R.STATUS_RANGE
    assert R.get_status() == 0
