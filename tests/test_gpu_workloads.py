"""GPU parity on the full-size workloads, in the launch configuration the benchmark uses:
caches written on the device by the library's write path, decode outputs compared with
the fp64 oracle decoding the same (device-written) records, write-path records compared
with the oracle on sampled tokens."""
import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import DECODE_TOL, META_TOL, SM_SCALE, bf16_bits, codes_match, f64, meta_match, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    R.lib()
    yield
    assert R.get_status() == 0


def _write_cache(w, layer, seq_lens, tau, gain, n_sink=0, n_recent=0, chunk=1 << 17, keep_rows=None):
    """Write every request's cache with the library (device latents, like the benchmark).
    keep_rows: {request: [positions]} whose latents are copied back for the oracle."""
    Rm = W.rotation(w.seed + layer)
    Rs = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    cache = R.PagedCache(int(pt.max()) + 1, torch.as_tensor(pt), n_sink, n_recent, device=DEV)
    cache.seq_lens = list(seq_lens)
    p = R.layer_params_init(tau, gain)
    lens = torch.as_tensor(seq_lens, dtype=torch.int32, device=DEV)
    kept = {}
    for b, L in enumerate(seq_lens):
        for s in range(0, L, chunk):
            n = min(chunk, L - s)
            c = W.latent_device(w, layer, n, DEV, stream=1000 + 97 * b + s // chunk)
            kr = W.rope_key_device(w, layer, n, DEV, stream=5000 + 97 * b + s // chunk)
            req = torch.full((n,), b, dtype=torch.int32, device=DEV)
            pos = torch.arange(s, s + n, dtype=torch.int32, device=DEV)
            R.quantize_append(cache, p, Rs, c, kr, req, pos, lens)
            if keep_rows and b in keep_rows:
                for q in keep_rows[b]:
                    if s <= q < s + n:
                        kept[(b, q)] = (c[q - s].cpu(), kr[q - s].cpu())
    torch.cuda.synchronize()
    return cache, p, Rm.astype(np.float64), pt, kept


def _decode_and_check(w, cache, p, pt, seq_lens, tau, heads, layer, reqs=None, n_sink=0, n_recent=0):
    B = len(seq_lens)
    q_c, q_r = W.queries(W.Workload(w.name, B, tuple(seq_lens), heads, seed=w.seed), layer)
    lens = torch.as_tensor(seq_lens, dtype=torch.int32, device=DEV)
    out, lse = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    torch.cuda.synchronize()
    out = out.cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    pool = cache.pages.cpu().numpy()
    prot = cache.prot.float().cpu().numpy().astype(np.float64) if cache.prot is not None else None
    worst = 0.0
    for r in (range(B) if reqs is None else reqs):
        L = seq_lens[r]
        packed, meta, kr = O.pages_read_fast(pool, pt, r, L)
        content = None
        if prot is not None:
            content = np.zeros((L, O.D_C))
            for pp in range(L):
                if pp < n_sink:
                    content[pp] = prot[r, pp]
                elif pp >= L - n_recent:
                    content[pp] = prot[r, n_sink + pp % n_recent]
        o, l = O.decode_request(f64(q_c[r]), f64(q_r[r]), packed, meta, O.bf16_bits_to_f64(kr), tau,
                                SM_SCALE, content, n_sink, n_recent)
        e = rel_l2(out[r], o).max()
        worst = max(worst, e)
        assert e <= DECODE_TOL, (r, e)
        assert np.abs(lse[r] - l).max() <= 1e-2 * max(1.0, np.abs(l).max())
    return worst


def _check_records(cache, pt, kept, Rm, tau, gain):
    pool = cache.pages.cpu().numpy()
    keys = sorted(kept)
    c = torch.stack([kept[k][0] for k in keys])
    kr = torch.stack([kept[k][1] for k in keys])
    q = O.quantize(f64(c), Rm, tau, gain)
    packed = np.stack([O.pages_read(pool, pt, b, pos + 1, start=pos)[0][0] for b, pos in keys])
    meta = np.stack([O.pages_read(pool, pt, b, pos + 1, start=pos)[1][0] for b, pos in keys])
    krb = np.stack([O.pages_read(pool, pt, b, pos + 1, start=pos)[2][0] for b, pos in keys])
    ok, frac, nbad = codes_match(packed, q, tau)
    assert ok, nbad
    emu, es = meta_match(meta, q, gain)
    assert emu <= META_TOL and es <= META_TOL, (emu, es)
    assert (krb == bf16_bits(kr)).all()
    if cache.prot is None:
        return
    # BF16 side store of protected positions: bf16(y) within one bf16 rounding of the oracle
    prot = cache.prot.float().cpu().numpy().astype(np.float64)
    L = {b: int(cache.seq_lens[b]) for b in range(cache.batch)}
    for i, (b, pos) in enumerate(keys):
        y = q["y"][i]
        if pos < cache.n_sink:
            slot = pos
        elif pos >= L[b] - cache.n_recent:
            slot = cache.n_sink + pos % cache.n_recent
        else:
            continue
        tol = np.abs(y) * 2.0 ** -7 + 1e-5 * np.abs(y).max()
        assert (np.abs(prot[b, slot] - y) <= tol).all(), (b, pos)


def test_decode_4x32k_one_layer():
    w = W.DECODE_4x32K
    tau, gain = W.layer_constants(w, 0)
    rng = np.random.default_rng(1)
    keep = {b: list(rng.choice(32768, 64, replace=False)) for b in range(4)}
    cache, p, Rm, pt, kept = _write_cache(w, 0, list(w.seq_lens), tau, gain, keep_rows=keep)
    _check_records(cache, pt, kept, Rm, tau, gain)
    worst = _decode_and_check(w, cache, p, pt, list(w.seq_lens), tau, 16, 0)
    print(f"\n4x32K decode worst rel-L2 {worst:.2e}")


@pytest.mark.slow
def test_decode_4x256k_27_layers_sampled():
    """All 27 layers written back to back as in the benchmark (each layer its own rotation,
    tau and gain); the oracle checks layers 0, 13 and 26 on every request."""
    w = W.DECODE_4x256K_27L
    checked = {}
    for layer in range(w.layers):
        tau, gain = W.layer_constants(w, layer)
        keep = {0: [0, 131071, 262143], 3: [1, 200000]} if layer in (0, 26) else None
        cache, p, Rm, pt, kept = _write_cache(w, layer, list(w.seq_lens), tau, gain, chunk=1 << 18,
                                              keep_rows=keep)
        if kept:
            _check_records(cache, pt, kept, Rm, tau, gain)
        if layer in (0, 13, 26):
            checked[layer] = (cache, p, tau)
    for layer, (cache, p, tau) in checked.items():
        worst = _decode_and_check(w, cache, p, W.page_table(w), list(w.seq_lens), tau, 16, layer)
        print(f"\n4x256K layer {layer} decode worst rel-L2 {worst:.2e}")


def test_decode_128_heads_paged_loguniform():
    w = W.PAGED_H128
    tau, gain = W.layer_constants(w, 0)
    cache, p, Rm, pt, _ = _write_cache(w, 0, list(w.seq_lens), tau, gain)
    worst = _decode_and_check(w, cache, p, pt, list(w.seq_lens), tau, 128, 0)
    print(f"\nH128 paged decode worst rel-L2 {worst:.2e} (lengths {min(w.seq_lens)}..{max(w.seq_lens)})")


def test_mixed_64x8k_sink4_recent128():
    w = W.MIXED_64x8K
    tau, gain = W.layer_constants(w, 0)
    rng = np.random.default_rng(2)
    keep = {b: [0, 3, 4, 8063, 8064, 8191] for b in rng.choice(64, 4, replace=False)}
    cache, p, Rm, pt, kept = _write_cache(w, 0, list(w.seq_lens), tau, gain, n_sink=4, n_recent=128,
                                          keep_rows=keep)
    _check_records(cache, pt, kept, Rm, tau, gain)
    worst = _decode_and_check(w, cache, p, pt, list(w.seq_lens), tau, 16, 0, reqs=range(0, 64, 3),
                              n_sink=4, n_recent=128)
    print(f"\n64x8K mixed decode worst rel-L2 {worst:.2e}")


def test_prefill_64k_sampled_layers():
    """The prefill write path (65,536 tokens per layer) on layers 0 and 26."""
    w = W.PREFILL_64K_27L
    rng = np.random.default_rng(3)
    for layer in (0, 26):
        tau, gain = W.layer_constants(w, layer)
        keep = {0: sorted(rng.choice(65536, 256, replace=False).tolist())}
        cache, p, Rm, pt, kept = _write_cache(w, layer, [65536], tau, gain, chunk=65536, keep_rows=keep)
        _check_records(cache, pt, kept, Rm, tau, gain)
