"""CPU oracle for the 2-bit rotated MLA cache (test infrastructure only).

Plain, slow, fp64 NumPy restatement of what the cache path computes, written from
"RoLaQ: Joint Rotation and Range Calibration for 2-Bit KV Caches in Multi-Head Latent
Attention" (arXiv 2610.20686v1) and the "2610.20686-rolaq-cache-accounting" notebook.
Only the tests, the package's smoke check and the benchmark's CPU-baseline leg may
import it; the library never does.  It shares no code with the CUDA path: the page
layout below is re-derived from the format description, not imported.

Readings taken where the pages leave a step open (each is listed with its reason in the
design notes):
  * rotation acts on row vectors, y = c . R, and y is kept at full precision (fp64
    here) until quantised;
  * group statistics are the mean and the population standard deviation (divide by
    128) of each 128-coordinate group, two-pass;
  * z = (y - mean) / std; code 0: z < -tau, 1: -tau <= z < 0, 2: 0 <= z < tau,
    3: z >= tau; a group with std == 0 takes z = 0 (code 2) and scale 0;
  * the four levels are -b, -a, +a, +b with a, b the centroids of a standard normal on
    [0, tau) and [tau, inf), computed in double and rounded to fp32 once;
  * metadata = (fp32(mean), fp32(gain * std)); reconstruction x = mean + scale * level;
  * decode: s = (q_c_rot . x + q_R . k_R) * sm_scale, softmax over the request's tokens,
    out = sum_t p_t x_t in the rotated basis, lse = log sum exp(s);
  * protected tokens (first n_sink, last n_recent) read bf16(y) instead of the codes.
Pins: every function here is pinned by tests against quadrature, closed forms,
brute force or the pages' printed numbers; none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

D_C = 512
D_R = 64
GROUP = 128
GROUPS = D_C // GROUP

# Storage accounting ("RoLaQ" §A.3; cache-accounting notebook): 2-bit codes for the 512
# content coordinates, two fp32 statistics per 128-group, a bf16 RoPE key.
CODE_BYTES = D_C * 2 // 8                  # 128
META_BYTES = GROUPS * 2 * 4                # 32
KR_BYTES = D_R * 2                         # 128
TOKEN_BYTES = CODE_BYTES + META_BYTES + KR_BYTES
BF16_TOKEN_BYTES = (D_C + D_R) * 2

# Page format of the cache pool (from the library's format description): 64 tokens per
# page, planes codes [64][128 B] | meta [64][4][2] fp32 | k_R [64][64] bf16.
PAGE_TOKENS = 64
PAGE_CODES = 0
PAGE_META = PAGE_CODES + PAGE_TOKENS * CODE_BYTES
PAGE_KR = PAGE_META + PAGE_TOKENS * META_BYTES
PAGE_BYTES = PAGE_KR + PAGE_TOKENS * KR_BYTES


# ---------------------------------------------------------------- quantizer levels --

def _phi(x: float) -> float:
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi(x: float) -> float:
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def levels(tau: float) -> Tuple[float, float]:
    """Inner and outer level (a, b) for threshold tau: conditional means of a standard
    normal on [0, tau) and [tau, inf).  §3.2 (threshold splits standardized coordinates
    into four levels), §C.3 / Fig. 8 (Lloyd-Max threshold)."""
    a = (_phi(0.0) - _phi(tau)) / (_Phi(tau) - 0.5)
    b = _phi(tau) / (1.0 - _Phi(tau))
    return a, b


def level_table(tau: float) -> np.ndarray:
    """Levels indexed by code 0..3, rounded to fp32 once: [-b, -a, +a, +b]."""
    a, b = levels(tau)
    return np.array([-b, -a, a, b], dtype=np.float32)


def lloyd_max_threshold(lo: float = 0.5, hi: float = 1.5, iters: int = 200) -> float:
    """Fixed point tau = (a(tau) + b(tau)) / 2 of the 4-level Lloyd-Max quantizer for a
    standard normal (the threshold OSCAR uses, Fig. 8; learned thresholds sit below it,
    §C.3).  Bisection on f(tau) = tau - (a + b) / 2."""
    def f(t):
        a, b = levels(t)
        return t - 0.5 * (a + b)
    flo = f(lo)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        fm = f(mid)
        if (fm < 0) == (flo < 0):
            lo, flo = mid, fm
        else:
            hi = mid
    return 0.5 * (lo + hi)


def response(tau: float, gain: float) -> float:
    """Response of the centered reconstruction, kappa = gain * E[z * level(z)] for
    z ~ N(0, 1) (§3.2 'unit response', §B.3).  With centroid levels
    E[z * level] = 2 * (a * (phi(0) - phi(tau)) + b * phi(tau))."""
    a, b = levels(tau)
    return gain * 2.0 * (a * (_phi(0.0) - _phi(tau)) + b * _phi(tau))


def coupled_gain(tau: float) -> float:
    """Gain giving unit response kappa = 1 (§3.2, §5.3)."""
    return 1.0 / response(tau, 1.0)


# ------------------------------------------------------------------- write path ----

def rotate(c: np.ndarray, R: np.ndarray) -> np.ndarray:
    """y = c . R in fp64 (§3.3: serving stores rotated latents)."""
    return np.asarray(c, np.float64) @ np.asarray(R, np.float64)


def group_stats(y: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per token and 128-group: mean and population std, two-pass ([T, 4] each)."""
    g = y.reshape(y.shape[0], GROUPS, GROUP)
    mu = g.mean(axis=2)
    sd = np.sqrt(((g - mu[:, :, None]) ** 2).mean(axis=2))
    return mu, sd


def standardize(y: np.ndarray, mu: np.ndarray, sd: np.ndarray) -> np.ndarray:
    """z = (y - mean) / std per group; z = 0 in a group with std == 0."""
    g = y.reshape(y.shape[0], GROUPS, GROUP)
    safe = np.where(sd > 0, sd, 1.0)
    z = (g - mu[:, :, None]) / safe[:, :, None]
    z = np.where(sd[:, :, None] > 0, z, 0.0)
    return z.reshape(y.shape)


def assign(z: np.ndarray, tau: float) -> np.ndarray:
    """Four-level assignment by threshold tau (§3.2), half-open intervals:
    0: z < -tau, 1: -tau <= z < 0, 2: 0 <= z < tau, 3: z >= tau."""
    t = np.float64(tau)
    codes = np.full(z.shape, 3, dtype=np.uint8)
    codes[z < t] = 2
    codes[z < 0.0] = 1
    codes[z < -t] = 0
    return codes


def pack(codes: np.ndarray) -> np.ndarray:
    """Four 2-bit codes per byte; coordinate j in bits 2*(j%4) of byte j//4."""
    c = codes.reshape(codes.shape[0], D_C // 4, 4).astype(np.uint32)
    out = c[:, :, 0] | (c[:, :, 1] << 2) | (c[:, :, 2] << 4) | (c[:, :, 3] << 6)
    return out.astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = packed.astype(np.uint32)
    parts = [(p >> (2 * k)) & 3 for k in range(4)]
    return np.stack(parts, axis=2).reshape(packed.shape[0], D_C).astype(np.uint8)


def quantize(c: np.ndarray, R: np.ndarray, tau: float, gain: float) -> dict:
    """Write path for T tokens: rotate, group statistics, standardise, assign, pack.
    Returns packed codes [T,128] u8, meta [T,4,2] fp32 (mean, gain*std), and the fp64
    intermediates y, z, mu, sd for comparisons."""
    y = rotate(c, R)
    mu, sd = group_stats(y)
    z = standardize(y, mu, sd)
    codes = assign(z, tau)
    meta = np.stack([mu.astype(np.float32), (np.float64(gain) * sd).astype(np.float32)],
                    axis=2)
    return {"y": y, "z": z, "mu": mu, "sd": sd, "codes": codes,
            "packed": pack(codes), "meta": meta}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even) and return as fp64.  The value is
    first rounded to fp32, which is how an fp32 pipeline reaches bf16."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(f)
    out = r.astype(np.uint32).view(np.float32).astype(np.float64)
    out[nan] = np.nan
    return out


# -------------------------------------------------------------------- read path ----

def dequantize(packed: np.ndarray, meta: np.ndarray, tau: float) -> np.ndarray:
    """x = mean_g + scale_g * level(code), fp64, from stored fp32 metadata and fp32
    levels (§3.2: the gain scales the reconstruction around the group mean)."""
    lv = level_table(tau).astype(np.float64)
    codes = unpack(packed)
    lev = lv[codes].reshape(-1, GROUPS, GROUP)
    mu = meta[:, :, 0].astype(np.float64)
    sc = meta[:, :, 1].astype(np.float64)
    return (mu[:, :, None] + sc[:, :, None] * lev).reshape(-1, D_C)


def attend(q_c_rot: np.ndarray, q_r: np.ndarray, x: np.ndarray, k_r: np.ndarray,
           sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Absorbed-MLA decode for one request: q_c_rot [H,512], q_r [H,64], x [T,512],
    k_r [T,64] -> out [H,512] (rotated basis), lse [H].  Scores
    (q_c_rot . x + q_r . k_r) * sm_scale, max-subtracted softmax over T (§3.3: the read
    side rotation is folded into the absorbed projections).  T == 0 -> zeros, -inf."""
    H = q_c_rot.shape[0]
    if x.shape[0] == 0:
        return np.zeros((H, D_C)), np.full(H, -np.inf)
    s = (np.asarray(q_c_rot, np.float64) @ x.T
         + np.asarray(q_r, np.float64) @ np.asarray(k_r, np.float64).T) * sm_scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    out = (e @ x) / l
    lse = (m + np.log(l))[:, 0]
    return out, lse


def protected_mask(L: int, n_sink: int, n_recent: int) -> np.ndarray:
    """Positions kept in bf16 (§4.1: first sink tokens and most recent tokens)."""
    p = np.arange(L)
    return (p < n_sink) | (p >= L - n_recent)


def decode_request(q_c_rot, q_r, packed, meta, k_r, tau, sm_scale,
                   prot_content: Optional[np.ndarray] = None,
                   n_sink: int = 0, n_recent: int = 0):
    """Decode one request from its logical cache arrays.  prot_content [L,512] holds the
    bf16 rotated content of each position (only protected positions are read)."""
    x = dequantize(packed, meta, tau)
    if prot_content is not None and (n_sink or n_recent):
        m = protected_mask(x.shape[0], n_sink, n_recent)
        x = x.copy()
        x[m] = prot_content[m]
    return attend(q_c_rot, q_r, x, k_r, sm_scale)


# ----------------------------------------------------------------- page format ----

def pages_write(pool: np.ndarray, page_table: np.ndarray, req: int, packed: np.ndarray,
                meta: np.ndarray, k_r_bits: np.ndarray, start: int = 0) -> None:
    """Place tokens start.. of request req into a uint8 page pool [num_pages*PAGE_BYTES].
    k_r_bits: uint16 bf16 bit patterns [T,64]."""
    T = packed.shape[0]
    meta_b = np.ascontiguousarray(meta.astype(np.float32)).view(np.uint8).reshape(T, META_BYTES)
    kr_b = np.ascontiguousarray(k_r_bits.astype(np.uint16)).view(np.uint8).reshape(T, KR_BYTES)
    for i in range(T):
        p = start + i
        base = int(page_table[req, p // PAGE_TOKENS]) * PAGE_BYTES
        row = p % PAGE_TOKENS
        pool[base + PAGE_CODES + row * CODE_BYTES: base + PAGE_CODES + (row + 1) * CODE_BYTES] = packed[i]
        pool[base + PAGE_META + row * META_BYTES: base + PAGE_META + (row + 1) * META_BYTES] = meta_b[i]
        pool[base + PAGE_KR + row * KR_BYTES: base + PAGE_KR + (row + 1) * KR_BYTES] = kr_b[i]


def pages_read(pool: np.ndarray, page_table: np.ndarray, req: int, L: int,
               start: int = 0):
    """Inverse of pages_write for positions start..L-1: (packed, meta fp32, k_R bits)."""
    n = L - start
    packed = np.empty((n, CODE_BYTES), np.uint8)
    meta = np.empty((n, META_BYTES), np.uint8)
    kr = np.empty((n, KR_BYTES), np.uint8)
    for i in range(n):
        p = start + i
        base = int(page_table[req, p // PAGE_TOKENS]) * PAGE_BYTES
        row = p % PAGE_TOKENS
        packed[i] = pool[base + PAGE_CODES + row * CODE_BYTES: base + PAGE_CODES + (row + 1) * CODE_BYTES]
        meta[i] = pool[base + PAGE_META + row * META_BYTES: base + PAGE_META + (row + 1) * META_BYTES]
        kr[i] = pool[base + PAGE_KR + row * KR_BYTES: base + PAGE_KR + (row + 1) * KR_BYTES]
    return packed, meta.view(np.float32).reshape(n, GROUPS, 2), kr.view(np.uint16).reshape(n, D_R)


def pages_read_fast(pool: np.ndarray, page_table: np.ndarray, req: int, L: int):
    """Vectorised pages_read for whole requests (same result, for large caches)."""
    npg = (L + PAGE_TOKENS - 1) // PAGE_TOKENS
    pages = pool.reshape(-1, PAGE_BYTES)[page_table[req, :npg].astype(np.int64)]
    codes = pages[:, PAGE_CODES:PAGE_META].reshape(-1, CODE_BYTES)[:L]
    meta = pages[:, PAGE_META:PAGE_KR].reshape(-1, META_BYTES)[:L]
    kr = pages[:, PAGE_KR:].reshape(-1, KR_BYTES)[:L]
    return (np.ascontiguousarray(codes),
            np.ascontiguousarray(meta).view(np.float32).reshape(L, GROUPS, 2),
            np.ascontiguousarray(kr).view(np.uint16).reshape(L, D_R))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) as fp64 values: a bfloat16 is the upper half of an
    IEEE fp32, so the pattern moves into bits 16..31 of a 32-bit word read as fp32."""
    return (np.asarray(bits, np.uint32) << 16).astype(np.uint32).view(np.float32).astype(np.float64)


# ---- absorbed projections around the cache (RoLaQ §3.3; Fig. 3a) -----------------
# In absorbed MLA, head h's no-RoPE key and value are k_h = c . W_UK[h] and
# v_h = c . W_UV[h] (c the 512-d content latent, W_* [512][128]).  A query's no-RoPE score
# q_h . k_h = (q_h . W_UK[h]^T) . c, and with the cache holding y = c . R (R orthogonal,
# c = y . R^T) this is (q_h . W_UK[h]^T . R) . y: the read-side rotation folds into the
# query projection.  The attention output over y, o_rot = sum_t p_t y_t, gives head h's
# value output sum_t p_t v_t = o_rot . R^T . W_UV[h]: the inverse rotation folds into the
# value projection.

def fold_weights(W_UK: np.ndarray, W_UV: np.ndarray, R: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """W_UK, W_UV [H][512][128], R [512][512] (y = c . R) -> W_q [H][128][512] = W_UK[h]^T . R
    and W_o [H][512][128] = R^T . W_UV[h], in fp64."""
    W_UK = np.asarray(W_UK, np.float64)
    W_UV = np.asarray(W_UV, np.float64)
    R = np.asarray(R, np.float64)
    W_q = np.stack([W_UK[h].T @ R for h in range(W_UK.shape[0])])
    W_o = np.stack([R.T @ W_UV[h] for h in range(W_UV.shape[0])])
    return W_q, W_o


def fold_query(q_nope: np.ndarray, W_q: np.ndarray) -> np.ndarray:
    """q_nope [B][H][128] -> q_c_rot [B][H][512] = q_nope[b,h] . W_q[h]."""
    q_nope = np.asarray(q_nope, np.float64)
    return np.einsum("bhn,hnj->bhj", q_nope, np.asarray(W_q, np.float64))


def unfold_output(out_rot: np.ndarray, W_o: np.ndarray) -> np.ndarray:
    """out_rot [B][H][512] (rotated basis) -> v [B][H][128] = out_rot[b,h] . W_o[h]."""
    return np.einsum("bhk,hkn->bhn", np.asarray(out_rot, np.float64), np.asarray(W_o, np.float64))
