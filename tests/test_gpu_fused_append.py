"""GPU parity of the serving step with the per-step write fused into the decode
(rolaq_decode_attn_append): each call appends token L - 1 of every request and decodes
over the cache that includes it.  Checked against the fp64 oracle step by step, and
against the separate calls (small append, then decode), whose records it must
reproduce bit for bit."""
import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import (DECODE_TOL, META_TOL, SM_SCALE, bf16_bits, codes_match, f64, meta_match,
                               rel_l2)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    R.lib()
    yield
    assert R.get_status() == 0


def _prefill(cache, p, R_split, lat, kr, L0):
    B = len(L0)
    lens = torch.as_tensor(L0, dtype=torch.int32).to(DEV)
    if sum(L0) == 0:
        return
    c = torch.cat([lat[r][:L0[r]] for r in range(B)]).to(DEV)
    k = torch.cat([kr[r][:L0[r]] for r in range(B)]).to(DEV)
    req = torch.cat([torch.full((L0[r],), r, dtype=torch.int32) for r in range(B)]).to(DEV)
    pos = torch.cat([torch.arange(L0[r], dtype=torch.int32) for r in range(B)]).to(DEV)
    R.quantize_append(cache, p, R_split, c, k, req, pos, lens)


def _oracle_step(cache, pt, lat, kr, Rm, lens, tau, gain, q_c, q_r, n_sink, n_recent, out, lse):
    """Check the records of every request against the oracle's write path, then the
    call's output against the oracle decode over those records."""
    pool = cache.pages.cpu().numpy()
    prot = cache.prot.float().cpu().numpy().astype(np.float64) if cache.prot is not None else None
    for r, L in enumerate(lens):
        if L == 0:
            assert (out[r] == 0).all() and np.isneginf(lse[r]).all()
            continue
        q = O.quantize(f64(lat[r][:L]), Rm, tau, gain)
        packed, meta, krb = O.pages_read_fast(pool, pt, r, L)
        ok, _, nbad = codes_match(packed, q, tau)
        assert ok, (r, L, nbad)
        emu, es = meta_match(meta, q, gain)
        assert emu <= META_TOL and es <= META_TOL, (r, emu, es)
        assert (krb == bf16_bits(kr[r][:L])).all()
        content = None
        if prot is not None:
            yb = O.bf16_round(q["y"])
            content = np.zeros((L, O.D_C))
            for pp in range(L):
                if pp < n_sink:
                    slot = pp
                elif n_recent and pp >= L - n_recent:
                    slot = n_sink + pp % n_recent
                else:
                    continue
                d = np.abs(prot[r, slot] - yb[pp])
                assert (d <= np.abs(yb[pp]) * 2.0 ** -7 + 1e-5 * np.abs(q["y"][pp]).max()).all(), (r, pp)
                content[pp] = prot[r, slot]
        o_ref, l_ref = O.decode_request(f64(q_c[r]), f64(q_r[r]), packed, meta, O.bf16_bits_to_f64(krb), tau,
                                        SM_SCALE, content, n_sink, n_recent)
        assert rel_l2(out[r], o_ref).max() <= DECODE_TOL, (r, L)
        assert np.abs(lse[r] - l_ref).max() <= 1e-2 * max(1.0, np.abs(l_ref).max()), (r, L)


@pytest.mark.parametrize("n_sink,n_recent", [(4, 16), (0, 0), (8, 0)])
def test_fused_append_streaming_matches_oracle(n_sink, n_recent):
    """Requests that start empty, at a page's last row and at a page boundary; one token
    per request per call for 20 calls; every call's records and output against the
    oracle.  (4, 16): the new token is always protected and the ring wraps; (0, 0): it is
    read from its codes; (8, 0): protected as a sink for the first calls only."""
    L0 = [0, 63, 64, 130, 5]
    steps = 20
    B = len(L0)
    tau, gain = 0.93, 1.11
    w = W.Workload("fused", B, tuple(l + steps for l in L0), 16, paged_shuffled=True, seed=311)
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    cache = R.PagedCache(int(pt.max() + 1), torch.as_tensor(pt), n_sink, n_recent, device=DEV)
    p = R.layer_params_init(tau, gain)
    Lf = [l + steps for l in L0]
    lat = [W.latent(w, 0, Lf[r], stream=100 + r) for r in range(B)]
    kr = [W.rope_key(w, 0, Lf[r], stream=200 + r) for r in range(B)]
    _prefill(cache, p, R_split, lat, kr, L0)
    ws = torch.empty(R.decode_append_workspace_bytes(B, 16), dtype=torch.uint8, device=DEV)
    for s in range(steps):
        lens_l = [L0[r] + s + 1 for r in range(B)]
        c = torch.stack([lat[r][L0[r] + s] for r in range(B)]).to(DEV)
        k = torch.stack([kr[r][L0[r] + s] for r in range(B)]).to(DEV)
        q_c, q_r = W.queries(w, s)
        lens = torch.as_tensor(lens_l, dtype=torch.int32).to(DEV)
        out, lse = R.decode_attn_append(cache, p, R_split, c, k, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE,
                                        workspace=ws)
        if s in (0, 1, 2, 7, 19):
            _oracle_step(cache, pt, lat, kr, Rm.astype(np.float64), lens_l, tau, gain, q_c, q_r, n_sink,
                         n_recent, out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64))


def _same_records(a, b):
    assert torch.equal(a.pages, b.pages)
    if a.prot is not None:
        assert torch.equal(a.prot.view(torch.int16), b.prot.view(torch.int16))


@pytest.mark.parametrize("heads", [16, 32, 48])
def test_fused_append_equals_separate_calls(heads):
    """Same starting cache, same new tokens: the fused call stores the records the small
    append stores (bit for bit, side store included) and its output matches the decode
    of the appended cache (the new token's score is summed in fp32 instead of on the
    tensor cores)."""
    L = [1, 64, 65, 777, 4096, 200]
    B = len(L)
    w = W.Workload("fused_eq", B, tuple(L), heads, paged_shuffled=True, n_sink=4, n_recent=32, seed=313)
    tau, gain = 0.9, 1.08
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    caches = [R.PagedCache(int(pt.max() + 1), torch.as_tensor(pt), 4, 32, device=DEV) for _ in range(2)]
    p = R.layer_params_init(tau, gain)
    lat = [W.latent(w, 0, L[r], stream=100 + r) for r in range(B)]
    kr = [W.rope_key(w, 0, L[r], stream=200 + r) for r in range(B)]
    L0 = [l - 1 for l in L]
    for cache in caches:
        _prefill(cache, p, R_split, lat, kr, L0)
    c = torch.stack([lat[r][L[r] - 1] for r in range(B)]).to(DEV)
    k = torch.stack([kr[r][L[r] - 1] for r in range(B)]).to(DEV)
    lens = torch.as_tensor(L, dtype=torch.int32).to(DEV)
    q_c, q_r = (t.to(DEV) for t in W.queries(w, 0))
    R.quantize_append(caches[0], p, R_split, c, k, torch.arange(B, dtype=torch.int32, device=DEV),
                      (lens - 1).contiguous(), lens)
    out_a, lse_a = R.decode_attn(caches[0], p, q_c, q_r, lens, SM_SCALE)
    out_b, lse_b = R.decode_attn_append(caches[1], p, R_split, c, k, q_c, q_r, lens, SM_SCALE)
    torch.cuda.synchronize()
    _same_records(caches[0], caches[1])
    oa, ob = out_a.cpu().numpy().astype(np.float64), out_b.cpu().numpy().astype(np.float64)
    assert rel_l2(ob, oa).max() <= 2e-3
    assert (lse_b - lse_a).abs().max().item() <= 2e-3


def test_fused_append_zero_length_requests_are_untouched():
    """A request of length 0 in the batch gets no record, out = 0 and lse = -inf; the
    others are appended and decoded."""
    L = [0, 10, 0, 3]
    B = len(L)
    w = W.Workload("fused_zero", B, (1, 10, 1, 3), 16, seed=317)
    tau, gain = 0.95, 1.1
    Rm = W.rotation(w.seed)
    R_split = R.prepare_rotation(torch.as_tensor(Rm).to(DEV))
    pt = W.page_table(w)
    cache = R.PagedCache(int(pt.max() + 1), torch.as_tensor(pt), device=DEV)
    cache.pages.fill_(0x5A)
    p = R.layer_params_init(tau, gain)
    lat = [W.latent(w, 0, max(L[r], 1), stream=100 + r) for r in range(B)]
    kr = [W.rope_key(w, 0, max(L[r], 1), stream=200 + r) for r in range(B)]
    _prefill(cache, p, R_split, lat, kr, [max(l - 1, 0) for l in L])
    c = torch.stack([lat[r][max(L[r] - 1, 0)] for r in range(B)]).to(DEV)
    k = torch.stack([kr[r][max(L[r] - 1, 0)] for r in range(B)]).to(DEV)
    q_c, q_r = W.queries(w, 0)
    lens = torch.as_tensor(L, dtype=torch.int32).to(DEV)
    out, lse = R.decode_attn_append(cache, p, R_split, c, k, q_c.to(DEV), q_r.to(DEV), lens, SM_SCALE)
    pool = cache.pages.cpu().numpy().reshape(-1, O.PAGE_BYTES)
    for r in (0, 2):
        assert (pool[pt[r, 0]] == 0x5A).all()
    _oracle_step(cache, pt, lat, kr, Rm.astype(np.float64), L, tau, gain, q_c, q_r, 0, 0,
                 out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64))


def test_fused_append_full_size_4x256k():
    """The serving step at 4 requests x 262,144 tokens (16 heads): the fused call and the
    separate calls agree on the records and the output, at the split plan the benchmark
    runs."""
    w = W.Workload("decode_4x256k_h16", 4, (262144,) * 4, 16, seed=4242)
    tau, gain = W.layer_constants(w, 0)
    p = R.layer_params_init(tau, gain)
    R_split = R.prepare_rotation(torch.as_tensor(W.rotation(w.seed)).to(DEV))
    pt = torch.as_tensor(W.page_table(w))
    caches = [R.PagedCache(int(pt.max()) + 1, pt, device=DEV) for _ in range(2)]
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=DEV)
    n = w.seq_lens[0] - 1
    for b in range(w.batch):
        c = W.latent_device(w, 0, n, DEV, stream=1000 + b)
        k = W.rope_key_device(w, 0, n, DEV, stream=5000 + b)
        req = torch.full((n,), b, dtype=torch.int32, device=DEV)
        pos = torch.arange(n, dtype=torch.int32, device=DEV)
        R.quantize_append(caches[0], p, R_split, c, k, req, pos, lens)
    caches[1].pages.copy_(caches[0].pages)
    c = W.latent_device(w, 0, w.batch, DEV, stream=9000)
    k = W.rope_key_device(w, 0, w.batch, DEV, stream=9001)
    g = torch.Generator(device=DEV)
    g.manual_seed(4242)
    q_c = torch.randn((w.batch, w.heads, R.D_C), generator=g, device=DEV).to(torch.bfloat16)
    q_r = torch.randn((w.batch, w.heads, R.D_R), generator=g, device=DEV).to(torch.bfloat16)
    R.quantize_append(caches[0], p, R_split, c, k, torch.arange(w.batch, dtype=torch.int32, device=DEV),
                      (lens - 1).contiguous(), lens)
    out_a, lse_a = R.decode_attn(caches[0], p, q_c, q_r, lens, SM_SCALE)
    out_b, lse_b = R.decode_attn_append(caches[1], p, R_split, c, k, q_c, q_r, lens, SM_SCALE)
    torch.cuda.synchronize()
    assert torch.equal(caches[0].pages, caches[1].pages)
    oa, ob = out_a.cpu().numpy().astype(np.float64), out_b.cpu().numpy().astype(np.float64)
    assert rel_l2(ob, oa).max() <= 2e-3
    assert (lse_b - lse_a).abs().max().item() <= 2e-3
