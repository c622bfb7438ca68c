"""Host-side pieces of the benchmark that read library output on the CPU: the unpacking
of codes and statistics used by the threshold sweep, checked against pages written by
the oracle's own page writer (consecutive pages of one request)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench                                   # noqa: E402
from oracle import rolaq_oracle as O           # noqa: E402


def test_sweep_unpackers_read_the_page_format():
    rng = np.random.default_rng(11)
    n = 150                                    # three pages, the last one partly filled
    c = rng.standard_normal((n, O.D_C))
    q = O.quantize(c, np.eye(O.D_C), 0.95, 1.07)
    npg = -(-n // O.PAGE_TOKENS)
    pool = np.zeros(npg * O.PAGE_BYTES, np.uint8)
    pt = np.arange(npg, dtype=np.int32)[None, :]
    O.pages_write(pool, pt, 0, q["packed"], q["meta"], np.zeros((n, O.D_R), np.uint16))
    codes = bench.unpack_codes(pool, n)
    assert codes.shape == (n, O.D_C)
    assert (codes == q["codes"]).all()
    meta = bench.unpack_meta(pool, n)
    assert (meta == q["meta"].astype(np.float32).astype(np.float64)).all()


def test_sweep_taus_include_the_reference_threshold():
    assert bench.LLOYD_MAX_TAU in bench.SWEEP_TAUS
    assert abs(O.lloyd_max_threshold() - bench.LLOYD_MAX_TAU) < 1e-3


def test_packed_host_buffers_round_trip():
    """The end-to-end leg moves each step's inputs and outputs as one packed buffer: every
    segment starts 256-byte aligned and reads back the tensor written into it."""
    import torch
    src = [torch.randn(4, 512).to(torch.bfloat16), torch.randn(4, 64).to(torch.bfloat16),
           torch.randn(4, 16, 512).to(torch.bfloat16), torch.randn(4, 16), torch.randn(3)]
    offs, total = bench.pack_offsets([(tuple(t.shape), t.dtype) for t in src])
    assert all(o % 256 == 0 for o, _, _, _ in offs)
    assert total >= sum(t.numel() * t.element_size() for t in src)
    buf = torch.zeros(total, dtype=torch.uint8)
    for v, t in zip(bench.pack_views(buf, offs), src):
        v.copy_(t)
    for v, t in zip(bench.pack_views(buf.clone(), offs), src):
        assert torch.equal(v, t)
