"""GPU parity of the absorbed projections around the cache (RoLaQ §3.3, Fig. 3a): the
weight fold, the per-step query fold and the output unfold, each against the fp64 oracle
with an error bound derived from the arithmetic, and the whole chain
fold -> decode -> unfold against the oracle's chain."""
import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import DECODE_TOL, SM_SCALE, build_oracle_cache, f64, oracle_decode, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda"
U32 = 2.0 ** -24          # fp32 unit roundoff
U_BF16 = 2.0 ** -8        # bf16 unit roundoff (8-bit significand)


def gamma(n):
    """Bound on the relative error of an n-term fp32 dot product accumulated with fma."""
    return n * U32 / (1 - n * U32)


def gamma_tc(n):
    """The same for tensor-core accumulation, whose additions may truncate instead of
    rounding to nearest: twice the unit roundoff per addition."""
    return 2 * gamma(n)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    R.lib()
    yield
    assert R.get_status() == 0


def _weights(seed, H):
    rng = np.random.default_rng([seed, 31])
    W_UK = (rng.standard_normal((H, O.D_C, 128)) / np.sqrt(O.D_C)).astype(np.float32)
    W_UV = (rng.standard_normal((H, O.D_C, 128)) / np.sqrt(O.D_C)).astype(np.float32)
    return W_UK, W_UV


@pytest.mark.parametrize("H", [16, 128])
def test_fold_weights_within_fp32_dot_bound(H):
    W_UK, W_UV = _weights(H, H)
    Rm = W.rotation(40 + H)
    W_q, W_o = R.fold_weights(torch.as_tensor(W_UK).to(DEV), torch.as_tensor(W_UV).to(DEV),
                              torch.as_tensor(Rm).to(DEV))
    torch.cuda.synchronize()
    W_q_ref, W_o_ref = O.fold_weights(W_UK, W_UV, Rm)
    aK, aV, aR = np.abs(W_UK.astype(np.float64)), np.abs(W_UV.astype(np.float64)), np.abs(Rm.astype(np.float64))
    bound_q = gamma(O.D_C) * np.stack([aK[h].T @ aR for h in range(H)]) + 1e-30
    bound_o = gamma(O.D_C) * np.stack([aR.T @ aV[h] for h in range(H)]) + 1e-30
    # fp32 sum, then one rounding to bf16
    bound_q = U_BF16 * (np.abs(W_q_ref) + bound_q) + bound_q
    bound_o = U_BF16 * (np.abs(W_o_ref) + bound_o) + bound_o
    eq = np.abs(f64(W_q) - W_q_ref)
    eo = np.abs(f64(W_o) - W_o_ref)
    assert (eq <= bound_q).all(), float((eq / bound_q).max())
    assert (eo <= bound_o).all(), float((eo / bound_o).max())
    # the rounding is to nearest: most entries are exactly bf16(ref)
    assert (f64(W_q) == f64(W.to_bf16(W_q_ref))).mean() > 0.99


@pytest.mark.parametrize("B,H", [(1, 16), (8, 16), (13, 16), (3, 128), (130, 16)])
def test_fold_query_within_bf16_rounding(B, H):
    rng = np.random.default_rng([B, H, 32])
    W_q = W.to_bf16(rng.standard_normal((H, 128, O.D_C)) / np.sqrt(128))
    q_nope = W.to_bf16(rng.standard_normal((B, H, 128)))
    out = R.fold_query(q_nope.to(DEV), W_q.to(DEV))
    torch.cuda.synchronize()
    qn, wq = f64(q_nope), f64(W_q)
    ref = O.fold_query(qn, wq)
    g = gamma_tc(128) * np.einsum("bhn,hnj->bhj", np.abs(qn), np.abs(wq))
    err = np.abs(f64(out) - ref)
    bound = U_BF16 * (np.abs(ref) + g) + g + 1e-30
    assert (err <= bound).all(), float((err / bound).max())


@pytest.mark.parametrize("B,H", [(1, 16), (8, 16), (11, 16), (2, 128), (70, 16)])
def test_unfold_output_within_bf16_input_bound(B, H):
    rng = np.random.default_rng([B, H, 33])
    W_o = W.to_bf16(rng.standard_normal((H, O.D_C, 128)) / np.sqrt(O.D_C))
    o = rng.standard_normal((B, H, O.D_C)).astype(np.float32)
    v = R.unfold_output(torch.as_tensor(o).to(DEV), W_o.to(DEV))
    torch.cuda.synchronize()
    wo = f64(W_o)
    ref = O.unfold_output(o, wo)
    # out is rounded to bf16 on the way into the product, then fp32 tensor-core sums
    s_abs = np.einsum("bhk,hkn->bhn", np.abs(o.astype(np.float64)), np.abs(wo))
    bound = U_BF16 * s_abs + gamma_tc(O.D_C) * (1 + U_BF16) * s_abs + 1e-30
    err = np.abs(v.cpu().numpy().astype(np.float64) - ref)
    assert (err <= bound).all(), float((err / bound).max())


def test_batch_zero_is_a_no_op():
    H = 16
    q = torch.zeros((0, H, 128), dtype=torch.bfloat16, device=DEV)
    assert R.fold_query(q, torch.zeros((H, 128, O.D_C), dtype=torch.bfloat16, device=DEV)).shape == (0, H, O.D_C)
    o = torch.zeros((0, H, O.D_C), dtype=torch.float32, device=DEV)
    assert R.unfold_output(o, torch.zeros((H, O.D_C, 128), dtype=torch.bfloat16, device=DEV)).shape == (0, H, 128)
    torch.cuda.synchronize()


def test_fold_decode_unfold_chain_matches_oracle_chain():
    """Un-rotated MLA inputs (q_nope, W_UK, W_UV) through fold -> packed-cache decode ->
    unfold on the GPU, against the oracle doing the same three steps in fp64."""
    w = W.Workload("chain", 3, (900, 64, 2049), 16, paged_shuffled=True, seed=96)
    lens_l = [900, 64, 2049]
    tau, gain, H = 0.95, 1.1, 16
    cache, data, Rm = build_oracle_cache(w, 0, lens_l, tau, gain, n_sink=4, n_recent=64)
    W_UK, W_UV = _weights(96, H)
    rng = np.random.default_rng([96, 34])
    q_nope = W.to_bf16(rng.standard_normal((3, H, 128)))
    q_r = W.to_bf16(rng.standard_normal((3, H, O.D_R)))
    lens = torch.as_tensor(lens_l, dtype=torch.int32).to(DEV)

    W_q, W_o = R.fold_weights(torch.as_tensor(W_UK).to(DEV), torch.as_tensor(W_UV).to(DEV),
                              torch.as_tensor(Rm.astype(np.float32)).to(DEV))
    q_c_rot = R.fold_query(q_nope.to(DEV), W_q)
    out, _ = R.decode_attn(cache, R.layer_params_init(tau, gain), q_c_rot, q_r.to(DEV), lens, SM_SCALE)
    v = R.unfold_output(out, W_o)
    torch.cuda.synchronize()

    W_q_ref, W_o_ref = O.fold_weights(W_UK, W_UV, Rm)
    qc_ref = O.fold_query(f64(q_nope), W_q_ref)
    o_ref, _ = oracle_decode(data, qc_ref, f64(q_r), lens_l, tau, SM_SCALE, 4, 64)
    v_ref = O.unfold_output(o_ref, W_o_ref)
    vg = v.cpu().numpy().astype(np.float64)
    for r in range(3):
        e = rel_l2(vg[r], v_ref[r])
        assert e.max() <= DECODE_TOL, (r, e.max())
