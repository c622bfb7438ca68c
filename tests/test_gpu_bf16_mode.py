"""GPU parity of the BF16 decode (rolaq_decode_attn_bf16): quantisation disabled, every
token read from its bf16 copy in the side store.  Against the fp64 oracle with every
token protected, and against this library's 2-bit-page decode on the same cache."""
import numpy as np
import pytest
import torch

from oracle import rolaq_oracle as O
from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import DECODE_TOL, SM_SCALE, build_oracle_cache, f64, oracle_decode, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    R.lib()
    yield
    assert R.get_status() == 0


@pytest.mark.parametrize("n_sink,n_recent,lens,heads", [
    (0, 192, (1, 63, 64, 65, 130, 192), 16),      # ragged pages, one request of one token
    (64, 128, (100, 192, 150, 64, 0), 32),        # sinks + ring, an empty request
    (0, 128, (128, 5), 48),                       # three 16-head chunks
])
def test_bf16_decode_matches_oracle(n_sink, n_recent, lens, heads):
    w = W.Workload("bf16mode", len(lens), tuple(lens), heads, paged_shuffled=True, n_sink=n_sink,
                   n_recent=n_recent, seed=331 + heads)
    tau, gain = 0.93, 1.1
    cache, data, _ = build_oracle_cache(w, 0, list(lens), tau, gain, n_sink, n_recent)
    p = R.layer_params_init(tau, gain)
    q_c, q_r = W.queries(w, 0)
    lens_t = torch.as_tensor(lens, dtype=torch.int32, device=DEV)
    out, lse = R.decode_attn_bf16(cache, p, q_c.to(DEV), q_r.to(DEV), lens_t, SM_SCALE)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_decode(data, f64(q_c), f64(q_r), list(lens), tau, SM_SCALE, n_sink, n_recent)
    out = out.cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    for r, L in enumerate(lens):
        if L == 0:
            assert (out[r] == 0).all() and np.isneginf(lse[r]).all()
            continue
        assert rel_l2(out[r], ref[r]).max() <= DECODE_TOL, r
        assert np.abs(lse[r] - ref_lse[r]).max() <= 1e-2 * max(1.0, np.abs(ref_lse[r]).max()), r
    # the same cache through the 2-bit-page decode (every token protected there too)
    out2, _ = R.decode_attn(cache, p, q_c.to(DEV), q_r.to(DEV), lens_t, SM_SCALE)
    out2 = out2.cpu().numpy().astype(np.float64)
    for r, L in enumerate(lens):
        if L:
            assert rel_l2(out[r], out2[r]).max() <= 5e-3, r


def test_bf16_decode_flags_tokens_without_a_copy():
    """A request longer than the sink and recent windows has positions without a bf16
    copy: the call sets ROLAQ_STATUS_BAD_SLOT (and reading the status clears it)."""
    lens = (200,)
    w = W.Workload("bf16bad", 1, lens, 16, n_sink=0, n_recent=128, seed=337)
    cache, _, _ = build_oracle_cache(w, 0, list(lens), 0.95, 1.0, 0, 128)
    p = R.layer_params_init(0.95, 1.0)
    q_c, q_r = W.queries(w, 0)
    R.decode_attn_bf16(cache, p, q_c.to(DEV), q_r.to(DEV), torch.as_tensor(lens, dtype=torch.int32, device=DEV),
                       SM_SCALE)
    torch.cuda.synchronize()
    assert R.get_status() & R.STATUS_BAD_SLOT
    assert R.get_status() == 0


def test_bf16_decode_full_size_4x256k():
    """The bench's BF16 comparison shape: 4 x 262,144 tokens at 16 heads, every token
    protected (written by the library's write path), against the 2-bit-page decode of the
    same cache, whose every token also reads the side store."""
    import bench
    w = W.Workload("bf16_full", 4, (262144,) * 4, 16, n_sink=0, n_recent=262144, seed=1010)
    lay = bench.DecodeLayer(w, 0, torch.device(DEV))
    lay.fill(w, 0, torch.device(DEV))
    lens = torch.as_tensor(w.seq_lens, dtype=torch.int32, device=DEV)
    out, lse = R.decode_attn_bf16(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE)
    out2, lse2 = R.decode_attn(lay.cache, lay.params, lay.q_c, lay.q_r, lens, SM_SCALE)
    torch.cuda.synchronize()
    a, b = out.cpu().numpy().astype(np.float64), out2.cpu().numpy().astype(np.float64)
    assert rel_l2(a, b).max() <= 5e-3
    assert (lse - lse2).abs().max().item() <= 1e-2
