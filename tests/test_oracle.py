"""Pins of the CPU oracle against quadrature, closed forms, brute force, library routines
and the numbers the RoLaQ pages print.  No GPU."""
import json
import math
import os
import statistics

import numpy as np
import pytest
import torch
from scipy import integrate, stats

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ levels -------

def centroids_by_quadrature(tau):
    pdf = stats.norm.pdf
    m_in = integrate.quad(lambda z: z * pdf(z), 0.0, tau)[0]
    p_in = integrate.quad(pdf, 0.0, tau)[0]
    m_out = integrate.quad(lambda z: z * pdf(z), tau, np.inf)[0]
    p_out = integrate.quad(pdf, tau, np.inf)[0]
    return m_in / p_in, m_out / p_out


@pytest.mark.parametrize("tau", [0.5, 0.85, 0.9816, 1.1, 1.7])
def test_levels_are_gaussian_centroids(tau):
    a, b = O.levels(tau)
    qa, qb = centroids_by_quadrature(tau)
    assert abs(a - qa) < 1e-10 and abs(b - qb) < 1e-10


def test_level_table_order_and_fp32():
    t = O.level_table(0.9)
    a, b = O.levels(0.9)
    assert t.dtype == np.float32
    assert list(t) == [np.float32(-b), np.float32(-a), np.float32(a), np.float32(b)]
    assert t[0] < t[1] < 0 < t[2] < t[3]


def test_lloyd_max_threshold_matches_max_1960():
    g = golden("lloyd_max_gaussian_4level.json")
    t = O.lloyd_max_threshold()
    a, b = O.levels(t)
    assert abs(t - g["t"]) < 0.5e-4
    assert abs(a - g["a"]) < 0.5e-4
    assert abs(b - g["b"]) < 0.5e-3
    # minimum MSE of the standardized reconstruction at g = 1: 1 - E[level^2]
    mse = 1.0 - O.response(t, 1.0)
    assert abs(mse - g["mse"]) < 0.5e-4
    # Lloyd-Max necessary condition: threshold midway between the levels
    assert abs(t - 0.5 * (a + b)) < 1e-9


def test_mse_optimal_response_is_about_088():
    g = golden("mse_optimal_response.json")
    t = O.lloyd_max_threshold()
    kappa = O.response(t, 1.0)
    assert abs(kappa - g["kappa"]) < g["tolerance"]
    # by quadrature: E[z * level(z)] with the centroid levels
    a, b = O.levels(t)
    pdf = stats.norm.pdf
    ez = 2 * (a * integrate.quad(lambda z: z * pdf(z), 0, t)[0]
              + b * integrate.quad(lambda z: z * pdf(z), t, np.inf)[0])
    assert abs(ez - kappa) < 1e-10
    # g = 1 minimises E[(z - g level)^2] for centroid levels: E[z level] / E[level^2] = 1
    el2 = 2 * (a * a * integrate.quad(pdf, 0, t)[0] + b * b * integrate.quad(pdf, t, np.inf)[0])
    assert abs(ez / el2 - 1.0) < 1e-9


def test_coupled_gain_gives_unit_response():
    for tau in (0.85, 0.9, 0.9816, 1.1):
        assert abs(O.response(tau, O.coupled_gain(tau)) - 1.0) < 1e-12
    assert abs(O.coupled_gain(O.lloyd_max_threshold()) - 1.1331) < 1e-4


def test_response_by_monte_carlo():
    rng = np.random.default_rng(5)
    z = rng.standard_normal(2_000_000)
    tau = 0.93
    lv = O.level_table(tau).astype(np.float64)
    ell = lv[O.assign(z, tau)]
    assert abs((z * ell).mean() - O.response(tau, 1.0)) < 3e-3


def test_stored_scale_is_gain_times_population_std():
    """Metadata is (mean, gain * population std) per group (RoLaQ §3.2: the gain scales the
    reconstruction around the group mean).  Closed forms with R = I: an arithmetic
    progression 0..127 has mean 63.5 and population std sqrt((128^2 - 1) / 12); an
    alternating +-1 group has mean 0 and std 1."""
    gain = 1.16
    c = np.zeros((1, 512))
    c[0, :128] = np.arange(128.0)
    c[0, 128:256] = np.where(np.arange(128) % 2 == 0, 1.0, -1.0)
    c[0, 256:384] = 3.0 * np.arange(128.0) - 7.0
    c[0, 384:] = np.where(np.arange(128) % 2 == 0, 0.25, -0.25)
    q = O.quantize(c, np.eye(512), 0.9816, gain)
    sd_ap = math.sqrt((128 ** 2 - 1) / 12.0)
    expect = [(63.5, gain * sd_ap), (0.0, gain), (3.0 * 63.5 - 7.0, gain * 3.0 * sd_ap), (0.0, gain * 0.25)]
    for gi, (mu, sc) in enumerate(expect):
        assert q["meta"][0, gi, 0] == np.float32(mu)
        assert q["meta"][0, gi, 1] == np.float32(sc)


def test_reconstruction_response_scales_with_gain():
    """For Gaussian latents the centered reconstruction (x - mean) / std has response
    E[z (x - mean) / std] = g * kappa(tau) (RoLaQ §3.2, §B.3): at tau = 0.9816 and g = 1.16,
    1.16 * 0.8825.  kappa by quadrature; Monte Carlo over 2,048,000 coordinates standardised
    within their 128-groups (the within-group standardisation moves the mean by well under
    the 1e-2 tolerance)."""
    tau, gain = 0.9816, 1.16
    rng = np.random.default_rng(11)
    c = rng.standard_normal((4000, 512))
    q = O.quantize(c, np.eye(512), tau, gain)
    x = O.dequantize(q["packed"], q["meta"], tau)
    y = q["y"].reshape(-1, 4, 128)
    mu, sd = q["mu"][:, :, None], q["sd"][:, :, None]
    z = (y - mu) / sd
    resp = (z * (x.reshape(-1, 4, 128) - mu) / sd).mean()
    qa, qb = centroids_by_quadrature(tau)
    pdf = stats.norm.pdf
    kappa = 2 * (qa * integrate.quad(lambda v: v * pdf(v), 0, tau)[0]
                 + qb * integrate.quad(lambda v: v * pdf(v), tau, np.inf)[0])
    assert abs(resp - gain * kappa) < 1e-2


def test_bf16_bits_decode_matches_torch():
    """bfloat16 bit patterns decode like torch's bfloat16 view (all non-NaN patterns of a
    random sample plus hand values: 0x3F80 = 1, 0xC000 = -2, 0x0001 = 2^-133, 0x7F7F the
    largest finite)."""
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 1 << 16, 20000).astype(np.uint16)
    bits = bits[~(((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0))]
    ref = torch.as_tensor(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_bits_to_f64(bits)
    assert (got == ref).all()
    hand = O.bf16_bits_to_f64(np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], np.uint16))
    assert list(hand) == [1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127]


# ------------------------------------------------------------- storage ----------

def test_storage_accounting_matches_pages():
    g = golden("storage_accounting.json")
    assert O.CODE_BYTES == g["code_bytes"]
    assert O.META_BYTES == g["metadata_bytes"]
    assert O.KR_BYTES == g["rope_bytes"]
    assert O.TOKEN_BYTES == g["total_bytes"]
    assert O.BF16_TOKEN_BYTES == g["bf16_bytes"]
    assert O.BF16_TOKEN_BYTES / O.TOKEN_BYTES == g["capacity_ceiling"]
    assert O.TOKEN_BYTES * 8 / (O.D_C + O.D_R) == g["effective_bits_per_coordinate"]
    # the measured ratio sits below the arithmetic ceiling (allocator overhead)
    assert g["measured_capacity_ratio"] < g["capacity_ceiling"]
    assert abs(g["rolaq_tokens_millions"] / g["bf16_tokens_millions"] - 3.96) < 0.01
    assert O.PAGE_BYTES == O.PAGE_TOKENS * O.TOKEN_BYTES == 18432


def test_header_constants_agree_with_oracle_layout():
    hdr = open(os.path.join(os.path.dirname(GOLDEN), "..", "include", "rolaq.h")).read()

    def val(name):
        import re
        m = re.search(r"#define\s+%s\s+(\d+)" % name, hdr)
        return int(m.group(1))
    assert val("ROLAQ_TOKEN_BYTES") == O.TOKEN_BYTES
    assert val("ROLAQ_PAGE_BYTES") == O.PAGE_BYTES
    assert val("ROLAQ_PAGE_META_OFFSET") == O.PAGE_META
    assert val("ROLAQ_PAGE_KR_OFFSET") == O.PAGE_KR
    assert val("ROLAQ_PAGE_TOKENS") == O.PAGE_TOKENS


# ------------------------------------------------------------ write path ---------

def test_bit_order_hand_example():
    g = golden("bit_order_example.json")
    codes = np.zeros((1, 512), np.uint8)
    codes[0, :8] = g["codes"]
    packed = O.pack(codes)
    assert list(packed[0, :2]) == g["bytes"]
    assert (O.unpack(packed) == codes).all()


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 4, size=(37, 512), dtype=np.uint8)
    p = O.pack(codes)
    assert p.shape == (37, 128)
    assert (O.unpack(p) == codes).all()
    # explicit bit arithmetic on one coordinate
    j = 301
    assert (((p[:, j // 4] >> (2 * (j % 4))) & 3) == codes[:, j]).all()


def test_assign_half_open_intervals():
    tau = 0.9
    eps = 1e-9
    z = np.array([-5, -tau - eps, -tau, -eps, 0.0, eps, tau - eps, tau, tau + eps, 5])
    assert list(O.assign(z, tau)) == [0, 0, 1, 1, 2, 2, 2, 3, 3, 3]


def test_group_stats_population_std():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((3, 512)) * 3 + 1
    mu, sd = O.group_stats(y)
    for t in range(3):
        for g in range(4):
            seg = list(y[t, 128 * g:128 * (g + 1)])
            assert abs(mu[t, g] - statistics.fmean(seg)) < 1e-12
            assert abs(sd[t, g] - statistics.pstdev(seg)) < 1e-12


def test_zero_spread_group():
    tau = 0.95
    c = np.zeros((1, 512))
    R = np.eye(512)
    c[0, :128] = 2.5                          # constant group 0
    c[0, 128:] = np.random.default_rng(2).standard_normal(384)
    q = O.quantize(c, R, tau, 1.1)
    assert (q["codes"][0, :128] == 2).all()
    assert q["meta"][0, 0, 0] == np.float32(2.5) and q["meta"][0, 0, 1] == 0.0
    x = O.dequantize(q["packed"], q["meta"], tau)
    assert (x[0, :128] == 2.5).all()


def test_rotation_is_orthogonal():
    R = W.rotation(1000).astype(np.float64)
    assert np.abs(R.T @ R - np.eye(512)).max() <= 1e-6
    # sign fix: the Gaussian's QR has a positive-diagonal triangular factor
    g = np.random.default_rng([1000, 77]).standard_normal((512, 512))
    assert np.abs(R @ (R.T @ g) - g).max() < 1e-4


def test_rotate_is_row_vector_product():
    rng = np.random.default_rng(3)
    c = rng.standard_normal((2, 512))
    R = rng.standard_normal((512, 512))
    y = O.rotate(c, R)
    j = 17
    assert abs(y[1, j] - sum(c[1, k] * R[k, j] for k in range(512))) < 1e-9


def test_code_frequencies_and_reconstruction_mse():
    rng = np.random.default_rng(4)
    tau = 0.9816
    c = rng.standard_normal((4000, 512))
    q = O.quantize(c, np.eye(512), tau, 1.0)
    freq = np.bincount(q["codes"].ravel(), minlength=4) / q["codes"].size
    p_out = 1 - stats.norm.cdf(tau)
    expect = [p_out, 0.5 - p_out, 0.5 - p_out, p_out]
    assert np.abs(freq - expect).max() < 0.01
    x = O.dequantize(q["packed"], q["meta"], tau)
    mse = (((x - q["y"]).reshape(-1, 4, 128) / q["sd"][:, :, None]) ** 2).mean()
    assert abs(mse - (1 - O.response(tau, 1.0))) < 0.01


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-8, 8, 10000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38]])
    ref = torch.as_tensor(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert (O.bf16_round(x) == ref).all()


# ------------------------------------------------------------- read path ---------

def brute_attend(q, qr, x, kr, scale):
    H, T = q.shape[0], x.shape[0]
    out = np.zeros((H, x.shape[1]))
    lse = np.zeros(H)
    for h in range(H):
        s = []
        for t in range(T):
            acc = 0.0
            for j in range(x.shape[1]):
                acc += q[h, j] * x[t, j]
            for j in range(kr.shape[1]):
                acc += qr[h, j] * kr[t, j]
            s.append(acc * scale)
        m = max(s)
        w = [math.exp(v - m) for v in s]
        tot = sum(w)
        for t in range(T):
            out[h] += (w[t] / tot) * x[t]
        lse[h] = m + math.log(tot)
    return out, lse


def test_attend_brute_force():
    rng = np.random.default_rng(7)
    H, T = 3, 6
    q = rng.standard_normal((H, 512)); qr = rng.standard_normal((H, 64))
    x = rng.standard_normal((T, 512)); kr = rng.standard_normal((T, 64))
    out, lse = O.attend(q, qr, x, kr, 1 / math.sqrt(192))
    bo, bl = brute_attend(q, qr, x, kr, 1 / math.sqrt(192))
    assert np.abs(out - bo).max() < 1e-12
    assert np.abs(lse - bl).max() < 1e-12


def test_dequantize_brute_force():
    rng = np.random.default_rng(8)
    tau = 0.88
    c = rng.standard_normal((3, 512)) * 2
    q = O.quantize(c, W.rotation(3).astype(np.float64), tau, 1.13)
    x = O.dequantize(q["packed"], q["meta"], tau)
    a, b = O.levels(tau)
    lv = [float(np.float32(-b)), float(np.float32(-a)), float(np.float32(a)), float(np.float32(b))]
    for t in range(3):
        for j in range(0, 512, 37):
            code = (int(q["packed"][t, j // 4]) >> (2 * (j % 4))) & 3
            g = j // 128
            ref = float(q["meta"][t, g, 0]) + float(q["meta"][t, g, 1]) * lv[code]
            assert x[t, j] == ref


def test_quantization_disabled_reduces_to_standard_mla():
    """With x = c . R stored exactly and the query folded (q . R), the rotated decode
    followed by the inverse rotation equals plain absorbed MLA on c (§3.3)."""
    rng = np.random.default_rng(9)
    H, T = 4, 40
    R = W.rotation(11).astype(np.float64)
    Rq, _ = np.linalg.qr(R)            # exactly orthogonal in fp64
    c = rng.standard_normal((T, 512)); kr = rng.standard_normal((T, 64))
    q = rng.standard_normal((H, 512)); qr = rng.standard_normal((H, 64))
    scale = 1 / math.sqrt(192)
    out_rot, lse_rot = O.attend(q @ Rq, qr, O.rotate(c, Rq), kr, scale)
    # plain MLA written out independently
    s = (q @ c.T + qr @ kr.T) * scale
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    ref = p @ c
    assert np.abs(out_rot @ Rq.T - ref).max() < 1e-12
    assert np.abs(lse_rot - np.log(np.exp(s).sum(1))).max() < 1e-12


def test_single_token_and_zero_query():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((1, 512)); kr = rng.standard_normal((1, 64))
    q = rng.standard_normal((2, 512)); qr = rng.standard_normal((2, 64))
    out, _ = O.attend(q, qr, x, kr, 0.1)
    assert np.abs(out - x[0]).max() < 1e-14
    x = rng.standard_normal((9, 512)); kr = rng.standard_normal((9, 64))
    out, lse = O.attend(np.zeros((2, 512)), np.zeros((2, 64)), x, kr, 0.1)
    assert np.abs(out - x.mean(0)).max() < 1e-14
    assert np.abs(lse - math.log(9)).max() < 1e-14


def test_empty_sequence():
    out, lse = O.attend(np.ones((2, 512)), np.ones((2, 64)), np.zeros((0, 512)),
                        np.zeros((0, 64)), 0.1)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_protected_positions():
    m = O.protected_mask(10, 2, 3)
    assert list(np.nonzero(m)[0]) == [0, 1, 7, 8, 9]
    m = O.protected_mask(4, 4, 128)
    assert m.all()
    rng = np.random.default_rng(11)
    L, tau = 12, 0.9
    c = rng.standard_normal((L, 512))
    q = O.quantize(c, np.eye(512), tau, 1.0)
    prot = O.bf16_round(q["y"])
    kr = rng.standard_normal((L, 64))
    qc = rng.standard_normal((2, 512)); qr = rng.standard_normal((2, 64))
    out, _ = O.decode_request(qc, qr, q["packed"], q["meta"], kr, tau, 0.1, prot, 2, 3)
    x = O.dequantize(q["packed"], q["meta"], tau)
    x[[0, 1, 9, 10, 11]] = prot[[0, 1, 9, 10, 11]]
    ref, _ = brute_attend(qc, qr, x, kr, 0.1)
    assert np.abs(out - ref).max() < 1e-12


def test_page_roundtrip_and_offsets():
    rng = np.random.default_rng(12)
    w = W.Workload("t", 2, (70, 130), 16, tau=0.9, gain=1.0, paged_shuffled=True, seed=5)
    pt = W.page_table(w)
    pool = np.zeros(int(pt.max() + 1) * O.PAGE_BYTES, np.uint8)
    data = {}
    for r, L in enumerate(w.seq_lens):
        packed = rng.integers(0, 256, (L, 128), dtype=np.uint8)
        meta = rng.standard_normal((L, 4, 2)).astype(np.float32)
        kr = rng.integers(0, 65536, (L, 64), dtype=np.uint16)
        O.pages_write(pool, pt, r, packed, meta, kr)
        data[r] = (packed, meta, kr)
    for r, L in enumerate(w.seq_lens):
        for a, b in zip(O.pages_read(pool, pt, r, L), data[r]):
            assert (a == b).all()
        for a, b in zip(O.pages_read_fast(pool, pt, r, L), data[r]):
            assert (a == b).all()
    # position 65 of request 1 sits in its second page, row 1
    page = pt[1, 1]
    assert (pool[page * 18432 + 128: page * 18432 + 256] == data[1][0][65]).all()
    assert (pool[page * 18432 + 8192 + 32: page * 18432 + 8192 + 64].view(np.float32)
            == data[1][1][65].ravel()).all()
    assert (pool[page * 18432 + 10240 + 128: page * 18432 + 10240 + 256].view(np.uint16)
            == data[1][2][65]).all()


# ------------------------------------------------ planted mistakes (oracle only) ----

def _pins_fail(monkeypatch, name, bad, pins):
    monkeypatch.setattr(O, name, bad)
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    return failed


def test_planted_mistakes_are_caught(monkeypatch):
    good_levels, good_stats, good_pack, good_assign = O.levels, O.group_stats, O.pack, O.assign

    def swapped_levels(tau):
        a, b = good_levels(tau)
        return b, a

    def sample_std(y):
        g = y.reshape(y.shape[0], 4, 128)
        return g.mean(2), g.std(2, ddof=1)

    def reversed_pack(codes):
        c = codes.reshape(codes.shape[0], 128, 4).astype(np.uint32)
        return (c[:, :, 3] | (c[:, :, 2] << 2) | (c[:, :, 1] << 4) | (c[:, :, 0] << 6)).astype(np.uint8)

    def closed_ties(z, tau):
        codes = np.full(z.shape, 3, dtype=np.uint8)
        codes[z <= tau] = 2
        codes[z <= 0.0] = 1
        codes[z <= -tau] = 0
        return codes

    cases = [
        ("levels", swapped_levels, [lambda: test_levels_are_gaussian_centroids(0.9)]),
        ("group_stats", sample_std, [test_group_stats_population_std]),
        ("pack", reversed_pack, [test_bit_order_hand_example]),
        ("assign", closed_ties, [test_assign_half_open_intervals]),
    ]
    for name, bad, pins in cases:
        with monkeypatch.context() as m:
            assert _pins_fail(m, name, bad, pins) == len(pins), name
    assert O.levels is good_levels and O.group_stats is good_stats
    assert O.pack is good_pack and O.assign is good_assign


def test_planted_gain_mistakes_are_caught(monkeypatch):
    """Dropping the gain from the stored scale, or applying it twice, fails both scale pins."""
    good = O.quantize
    pins = [test_stored_scale_is_gain_times_population_std, test_reconstruction_response_scales_with_gain]
    for bad in (lambda c, R, tau, gain: good(c, R, tau, 1.0),
                lambda c, R, tau, gain: good(c, R, tau, gain * gain)):
        with monkeypatch.context() as m:
            assert _pins_fail(m, "quantize", bad, pins) == len(pins)
    assert O.quantize is good


def test_planted_bf16_decode_mistake_is_caught(monkeypatch):
    """A wrong shift in the bfloat16 bit decode fails its pin."""
    bad = lambda bits: (np.asarray(bits, np.uint32) << 15).astype(np.uint32).view(np.float32).astype(np.float64)
    with monkeypatch.context() as m:
        assert _pins_fail(m, "bf16_bits_to_f64", bad, [test_bf16_bits_decode_matches_torch]) == 1


def test_planted_transposed_rotation_is_caught(monkeypatch):
    monkeypatch.setattr(O, "rotate", lambda c, R: np.asarray(c, np.float64) @ np.asarray(R, np.float64).T)
    with pytest.raises(AssertionError):
        test_quantization_disabled_reduces_to_standard_mla()


# ---- absorbed projections (query fold / output unfold) ----------------------------

def _mla_weights(seed, H=4):
    rng = np.random.default_rng(seed)
    W_UK = rng.standard_normal((H, O.D_C, 128)) / math.sqrt(O.D_C)
    W_UV = rng.standard_normal((H, O.D_C, 128)) / math.sqrt(O.D_C)
    q, r = np.linalg.qr(rng.standard_normal((O.D_C, O.D_C)))
    return W_UK, W_UV, q * np.sign(np.diag(r))[None, :]


def test_fold_query_preserves_no_rope_scores():
    """q . (c W_UK)^T must equal fold(q) . (c R)^T for every token: the fold is exactly the
    read-side rotation absorbed into the query projection."""
    W_UK, W_UV, R = _mla_weights(3)
    rng = np.random.default_rng(4)
    c = rng.standard_normal((50, O.D_C))
    q = rng.standard_normal((2, 4, 128))
    W_q, _ = O.fold_weights(W_UK, W_UV, R)
    qt = O.fold_query(q, W_q)
    y = O.rotate(c, R)
    for b in range(2):
        for h in range(4):
            direct = q[b, h] @ (c @ W_UK[h]).T
            folded = qt[b, h] @ y.T
            assert np.allclose(folded, direct, rtol=1e-12, atol=1e-12)


def test_unfold_output_recovers_values():
    """sum_t p_t (c_t W_UV) must equal unfold(sum_t p_t y_t)."""
    W_UK, W_UV, R = _mla_weights(5)
    rng = np.random.default_rng(6)
    c = rng.standard_normal((40, O.D_C))
    p = rng.dirichlet(np.ones(40), size=(2, 4))          # [2][4][40] attention weights
    y = O.rotate(c, R)
    _, W_o = O.fold_weights(W_UK, W_UV, R)
    out_rot = np.einsum("bht,tk->bhk", p, y)
    v = O.unfold_output(out_rot, W_o)
    for b in range(2):
        for h in range(4):
            assert np.allclose(v[b, h], p[b, h] @ (c @ W_UV[h]), rtol=1e-12, atol=1e-12)


def test_fold_with_identity_rotation_is_transpose():
    W_UK, W_UV, _ = _mla_weights(7, H=2)
    W_q, W_o = O.fold_weights(W_UK, W_UV, np.eye(O.D_C))
    assert np.array_equal(W_q, np.transpose(W_UK, (0, 2, 1)))
    assert np.array_equal(W_o, W_UV)


def test_planted_fold_mistake_is_caught(monkeypatch):
    """Folding R^T instead of R into the query breaks the score identity."""
    W_UK, W_UV, R = _mla_weights(8, H=1)
    orig = O.fold_weights
    monkeypatch.setattr(O, "fold_weights", lambda a, b, r: orig(a, b, np.asarray(r).T))
    rng = np.random.default_rng(9)
    c = rng.standard_normal((10, O.D_C))
    q = rng.standard_normal((1, 1, 128))
    W_q, _ = O.fold_weights(W_UK, W_UV, R)
    folded = O.fold_query(q, W_q)[0, 0] @ O.rotate(c, R).T
    direct = q[0, 0] @ (c @ W_UK[0]).T
    assert not np.allclose(folded, direct, rtol=1e-6, atol=1e-6)
