"""rolaq_decode_attn_static: decode for callers that cannot allocate device memory (a
memory pool or captured allocator owns the device, a plug-in gets tensors but no
allocator, a host forbids allocation after start-up).  Its split-K scratch is a fixed
array inside the library; this checks it against rolaq_decode_attn, which uses caller
workspace, on two calls in a row with different inputs, through the C ABI.

Kept in its own file that sorts last, so a run that stops at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from decode_attention_rotate_b200 import rolaq as R
from decode_attention_rotate_b200 import workloads as W
from tests.gpu_helpers import DECODE_TOL, SM_SCALE, build_oracle_cache, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(seed, lens, heads, tau, gain, n_sink=0, n_recent=0):
    w = W.Workload(f"na{seed}", len(lens), tuple(lens), heads, paged_shuffled=True, seed=seed)
    cache, _, _ = build_oracle_cache(w, 0, lens, tau, gain, n_sink, n_recent)
    q_c, q_r = W.queries(w, 0)
    p = R.layer_params_init(tau, gain)
    return cache, p, q_c.to(DEV), q_r.to(DEV), torch.as_tensor(lens, dtype=torch.int32).to(DEV)


def test_static_scratch_decode_matches_workspace_decode_twice():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    cases = [
        _case(301, [3000, 65, 1], 16, 0.95, 1.1),
        _case(302, [1024, 2048], 128, 0.88, 1.05, n_sink=4, n_recent=128),
    ]
    for cache, p, q_c, q_r, lens in cases:
        ref, ref_lse = R.decode_attn(cache, p, q_c, q_r, lens, SM_SCALE)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        R.decode_attn_static(cache, p, q_c, q_r, lens, SM_SCALE, out, lse)
        torch.cuda.synchronize()
        a = out.cpu().numpy().astype(np.float64)
        b = ref.cpu().numpy().astype(np.float64)
        for r in range(a.shape[0]):
            assert rel_l2(a[r], b[r]).max() <= DECODE_TOL
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= 1e-3
    assert R.get_status() == 0


def test_static_scratch_rejects_oversized_requests():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    cache, p, q_c, q_r, lens = _case(303, [64], 16, 0.9, 1.0)
    # 128 heads x 1000 requests needs far more split-K scratch than the fixed array holds
    need = R.decode_workspace_bytes(1000, 128)
    assert need > R.STATIC_SCRATCH_BYTES
    big_q = torch.zeros((1000, 128, 512), dtype=torch.bfloat16, device=DEV)
    big_r = torch.zeros((1000, 128, 64), dtype=torch.bfloat16, device=DEV)
    # a batch beyond the cache's is an argument error, checked first
    with pytest.raises(R.RolaqError) as e:
        R.decode_attn_static(cache, p, big_q, big_r, lens, SM_SCALE)
    assert e.value.code == -1
    # a cache of 1000 requests (all on one page; nothing is launched): no room for the plan
    wide = R.PagedCache(cache.num_pages, torch.zeros((1000, 1), dtype=torch.int32), device=DEV, pages=cache.pages)
    with pytest.raises(R.RolaqError) as e:
        R.decode_attn_static(wide, p, big_q, big_r, lens, SM_SCALE)
    assert e.value.code == -2
