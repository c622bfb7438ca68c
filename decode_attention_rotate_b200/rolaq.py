"""Python binding of librolaq (argument marshalling only).

Every function forwards to the C entry point of the same name in librolaq.so; all
computation happens in the library's CUDA kernels.  Tensors are torch CUDA tensors
(PyTorch provides device memory and streams here).  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

from . import build as _build

D_C = 512
D_R = 64
D_NOPE = 128            # per-head no-RoPE query width
D_V = 128               # per-head value width
GROUP = 128              # coordinates per quantization group
GROUPS = 4
CODE_BYTES = 128         # 512 x 2 bit per token
META_BYTES = 32          # 4 groups x (mean, scale) fp32
PAGE_TOKENS = 64
PAGE_BYTES = 18432
TOKEN_BYTES = 288
BF16_TOKEN_BYTES = 1152   # uncompressed MLA record: (512 + 64) x bf16
RSPLIT_BYTES = 3 * 512 * 512 * 2

STATUS_BAD_PAGE = 1
STATUS_BAD_SLOT = 2
STATUS_TIMEOUT = 4
STATUS_RANGE = 8


class RolaqError(RuntimeError):
    """A C-ABI call returned a negative code; `code` holds it (ROLAQ_E* of rolaq.h)."""

    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({strerror(code)})")
        self.code = code


class rolaq_cache(ctypes.Structure):
    """The C descriptor of one layer's paged cache (struct rolaq_cache of rolaq.h)."""
    _fields_ = [
        ("pages_dev", ctypes.c_void_p),
        ("num_pages", ctypes.c_int64),
        ("page_table_dev", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("prot_dev", ctypes.c_void_p),
        ("n_sink", ctypes.c_int32),
        ("n_recent", ctypes.c_int32),
    ]


class rolaq_layer_params(ctypes.Structure):
    """Per-layer constants: threshold tau, gain, and the reconstruction levels a, b."""
    _fields_ = [
        ("tau", ctypes.c_float),
        ("gain", ctypes.c_float),
        ("level_a", ctypes.c_float),
        ("level_b", ctypes.c_float),
    ]


_LIB = None


def library_path() -> str:
    """Path of the in-tree librolaq.so."""
    return _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library with its prototypes; raises when it has not been built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"librolaq.so not built ({path}); run decode_attention_rotate_b200.build")
        L = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        P = ctypes.POINTER
        L.rolaq_version.restype = i32
        L.rolaq_strerror.restype = ctypes.c_char_p
        L.rolaq_strerror.argtypes = [i32]
        L.rolaq_coupled_gain.restype = i32
        L.rolaq_coupled_gain.argtypes = [ctypes.c_float, P(ctypes.c_double), P(ctypes.c_double)]
        L.rolaq_layer_params_init.restype = i32
        L.rolaq_layer_params_init.argtypes = [P(rolaq_layer_params), ctypes.c_float, ctypes.c_float]
        L.rolaq_prepare_rotation.restype = i32
        L.rolaq_prepare_rotation.argtypes = [vp, vp, vp]
        L.rolaq_quantize_append.restype = i32
        L.rolaq_quantize_append.argtypes = [P(rolaq_cache), P(rolaq_layer_params), vp, vp, vp, vp, vp,
                                            vp, i32, vp]
        L.rolaq_decode_workspace_bytes.restype = sz
        L.rolaq_decode_workspace_bytes.argtypes = [i32, i32]
        L.rolaq_decode_attn.restype = i32
        L.rolaq_decode_attn.argtypes = [P(rolaq_cache), P(rolaq_layer_params), vp, vp, vp, i32, i32,
                                        ctypes.c_float, vp, vp, vp, sz, vp]
        L.rolaq_decode_attn_bf16.restype = i32
        L.rolaq_decode_attn_bf16.argtypes = [P(rolaq_cache), P(rolaq_layer_params), vp, vp, vp, i32, i32,
                                             ctypes.c_float, vp, vp, vp, sz, vp]
        L.rolaq_decode_append_workspace_bytes.restype = sz
        L.rolaq_decode_append_workspace_bytes.argtypes = [i32, i32]
        L.rolaq_decode_attn_append.restype = i32
        L.rolaq_decode_attn_append.argtypes = [P(rolaq_cache), P(rolaq_layer_params), vp, vp, vp, vp, vp, vp,
                                               i32, i32, ctypes.c_float, vp, vp, vp, sz, vp]
        L.rolaq_decode_attn_static.restype = i32
        L.rolaq_decode_attn_static.argtypes = [P(rolaq_cache), P(rolaq_layer_params), vp, vp, vp, i32, i32,
                                               ctypes.c_float, vp, vp, vp]
        L.rolaq_fold_weights.restype = i32
        L.rolaq_fold_weights.argtypes = [vp, vp, vp, i32, vp, vp, vp]
        L.rolaq_fold_query.restype = i32
        L.rolaq_fold_query.argtypes = [vp, vp, i32, i32, vp, vp]
        L.rolaq_unfold_output.restype = i32
        L.rolaq_unfold_output.argtypes = [vp, vp, i32, i32, vp, vp]
        L.rolaq_get_status.restype = i32
        L.rolaq_get_status.argtypes = [P(ctypes.c_int), vp]
        _LIB = L
    return _LIB


def header_functions() -> list:
    """Names of the functions include/rolaq.h declares."""
    hdr = os.path.join(_build.INCLUDE, "rolaq.h")
    text = open(hdr).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rolaq_[a-z_0-9]+)\s*\(", text)))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise RolaqError(fn, rc)


def version() -> int:
    """rolaq_version: major * 10000 + minor * 100 + patch."""
    return lib().rolaq_version()


def strerror(code: int) -> str:
    """rolaq_strerror: static description of an error code."""
    return lib().rolaq_strerror(code).decode()


def coupled_gain(tau: float):
    """rolaq_coupled_gain: (gain giving unit response at threshold tau, E[z level(z)])."""
    g, k = ctypes.c_double(), ctypes.c_double()
    _check("rolaq_coupled_gain", lib().rolaq_coupled_gain(tau, ctypes.byref(g), ctypes.byref(k)))
    return g.value, k.value


def layer_params_init(tau: float, gain: float) -> rolaq_layer_params:
    """rolaq_layer_params_init: the levels a(tau), b(tau) computed in double, stored fp32."""
    p = rolaq_layer_params()
    _check("rolaq_layer_params_init", lib().rolaq_layer_params_init(ctypes.byref(p), tau, gain))
    return p


def prepare_rotation(R: torch.Tensor, R_split: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """R: fp32 [512, 512] CUDA (y = c @ R).  Returns the bf16 operand [3, 512, 512]."""
    assert R.dtype == torch.float32 and tuple(R.shape) == (D_C, D_C)
    if R_split is None:
        R_split = torch.empty((3, D_C, D_C), dtype=torch.bfloat16, device=R.device)
    _check("rolaq_prepare_rotation", lib().rolaq_prepare_rotation(_ptr(R), _ptr(R_split), _stream(stream)))
    return R_split


class PagedCache:
    """Device buffers of one layer's cache plus the C descriptor that points at them."""

    def __init__(self, num_pages: int, page_table: torch.Tensor, n_sink: int = 0, n_recent: int = 0,
                 device="cuda", pages: Optional[torch.Tensor] = None):
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.batch, self.max_pages = self.page_table.shape
        self.num_pages = int(num_pages)
        self.pages = pages if pages is not None else torch.zeros(
            self.num_pages * PAGE_BYTES, dtype=torch.uint8, device=device)
        self.n_sink, self.n_recent = int(n_sink), int(n_recent)
        nslot = self.n_sink + self.n_recent
        self.prot = (torch.zeros((self.batch, nslot, D_C), dtype=torch.bfloat16, device=device)
                     if nslot else None)

    def desc(self) -> rolaq_cache:
        c = rolaq_cache()
        c.pages_dev = _ptr(self.pages)
        c.num_pages = self.num_pages
        c.page_table_dev = _ptr(self.page_table)
        c.batch = self.batch
        c.max_pages_per_seq = self.max_pages
        c.prot_dev = _ptr(self.prot) if self.prot is not None else None
        c.n_sink = self.n_sink
        c.n_recent = self.n_recent
        return c


def quantize_append(cache: PagedCache, params: rolaq_layer_params, R_split: torch.Tensor,
                    c: torch.Tensor, k_r: torch.Tensor, req: torch.Tensor, pos: torch.Tensor,
                    seq_lens: Optional[torch.Tensor] = None, stream=None) -> None:
    """rolaq_quantize_append: write the 2-bit records of n tokens (c bf16 [n, 512], k_r
    bf16 [n, 64]) at (req[i], pos[i]); seq_lens (request lengths after the append) is
    needed when the cache has a recent window."""
    n = int(c.shape[0])
    assert c.dtype == torch.bfloat16 and k_r.dtype == torch.bfloat16
    assert req.dtype == torch.int32 and pos.dtype == torch.int32
    d = cache.desc()
    _check("rolaq_quantize_append", lib().rolaq_quantize_append(
        ctypes.byref(d), ctypes.byref(params), _ptr(R_split), _ptr(c), _ptr(k_r), _ptr(req), _ptr(pos),
        _ptr(seq_lens), n, _stream(stream)))


def decode_workspace_bytes(batch: int, heads: int) -> int:
    """rolaq_decode_workspace_bytes: split-K scratch rolaq_decode_attn needs."""
    return int(lib().rolaq_decode_workspace_bytes(batch, heads))


def decode_attn(cache: PagedCache, params: rolaq_layer_params, q_c_rot: torch.Tensor, q_r: torch.Tensor,
                seq_lens: torch.Tensor, sm_scale: float, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream=None):
    """rolaq_decode_attn: q_c_rot bf16 [B, H, 512] (rotation folded in), q_r bf16 [B, H, 64]
    -> (out fp32 [B, H, 512] in the rotated basis, lse fp32 [B, H]); allocates out, lse
    and the workspace when they are not given."""
    B, H = int(q_c_rot.shape[0]), int(q_c_rot.shape[1])
    assert q_c_rot.dtype == torch.bfloat16 and q_r.dtype == torch.bfloat16
    dev = q_c_rot.device
    if out is None:
        out = torch.empty((B, H, D_C), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    nbytes = decode_workspace_bytes(B, H)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    d = cache.desc()
    _check("rolaq_decode_attn", lib().rolaq_decode_attn(
        ctypes.byref(d), ctypes.byref(params), _ptr(q_c_rot), _ptr(q_r), _ptr(seq_lens), B, H,
        float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def decode_attn_bf16(cache: PagedCache, params: rolaq_layer_params, q_c_rot: torch.Tensor, q_r: torch.Tensor,
                     seq_lens: torch.Tensor, sm_scale: float, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                     stream=None):
    """rolaq_decode_attn_bf16: decode from the bf16 side store (every token protected);
    arguments and result as decode_attn."""
    B, H = int(q_c_rot.shape[0]), int(q_c_rot.shape[1])
    assert q_c_rot.dtype == torch.bfloat16 and q_r.dtype == torch.bfloat16
    dev = q_c_rot.device
    if out is None:
        out = torch.empty((B, H, D_C), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(decode_workspace_bytes(B, H), 16), dtype=torch.uint8, device=dev)
    d = cache.desc()
    _check("rolaq_decode_attn_bf16", lib().rolaq_decode_attn_bf16(
        ctypes.byref(d), ctypes.byref(params), _ptr(q_c_rot), _ptr(q_r), _ptr(seq_lens), B, H,
        float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def decode_append_workspace_bytes(batch: int, heads: int) -> int:
    """rolaq_decode_append_workspace_bytes: scratch rolaq_decode_attn_append needs."""
    return int(lib().rolaq_decode_append_workspace_bytes(batch, heads))


def decode_attn_append(cache: PagedCache, params: rolaq_layer_params, R_split: torch.Tensor,
                       c_new: torch.Tensor, k_r_new: torch.Tensor, q_c_rot: torch.Tensor, q_r: torch.Tensor,
                       seq_lens: torch.Tensor, sm_scale: float, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None):
    """rolaq_decode_attn_append: append token seq_lens[r] - 1 of every request r (c_new bf16
    [B, 512], k_r_new bf16 [B, 64]) and decode over the cache that includes it; returns
    (out, lse) as decode_attn."""
    B, H = int(q_c_rot.shape[0]), int(q_c_rot.shape[1])
    assert q_c_rot.dtype == torch.bfloat16 and q_r.dtype == torch.bfloat16
    assert c_new.dtype == torch.bfloat16 and k_r_new.dtype == torch.bfloat16
    assert tuple(c_new.shape) == (B, D_C) and tuple(k_r_new.shape) == (B, D_R)
    assert c_new.is_contiguous() and k_r_new.is_contiguous()
    dev = q_c_rot.device
    if out is None:
        out = torch.empty((B, H, D_C), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(decode_append_workspace_bytes(B, H), 16), dtype=torch.uint8, device=dev)
    d = cache.desc()
    _check("rolaq_decode_attn_append", lib().rolaq_decode_attn_append(
        ctypes.byref(d), ctypes.byref(params), _ptr(R_split), _ptr(c_new), _ptr(k_r_new), _ptr(q_c_rot),
        _ptr(q_r), _ptr(seq_lens), B, H, float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return out, lse


STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


def decode_attn_static(cache: PagedCache, params: rolaq_layer_params, q_c_rot: torch.Tensor,
                       q_r: torch.Tensor, seq_lens: torch.Tensor, sm_scale: float,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       stream=None):
    """rolaq_decode_attn_static: decode with the library's own scratch array, for callers
    that cannot allocate device memory.  out / lse must be passed by such callers (the
    defaults here allocate them for convenience)."""
    B, H = int(q_c_rot.shape[0]), int(q_c_rot.shape[1])
    assert q_c_rot.dtype == torch.bfloat16 and q_r.dtype == torch.bfloat16
    assert tuple(q_c_rot.shape) == (B, H, D_C) and tuple(q_r.shape) == (B, H, D_R)
    dev = q_c_rot.device
    if out is None:
        out = torch.empty((B, H, D_C), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    assert out.dtype == torch.float32 and out.is_contiguous() and tuple(out.shape) == (B, H, D_C)
    assert lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, H)
    d = cache.desc()
    _check("rolaq_decode_attn_static", lib().rolaq_decode_attn_static(
        ctypes.byref(d), ctypes.byref(params), _ptr(q_c_rot), _ptr(q_r), _ptr(seq_lens), B, H,
        float(sm_scale), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def fold_weights(W_UK: torch.Tensor, W_UV: torch.Tensor, R: torch.Tensor, stream=None):
    """rolaq_fold_weights: W_UK, W_UV fp32 [H, 512, 128], R fp32 [512, 512] ->
    (W_q bf16 [H, 128, 512], W_o bf16 [H, 512, 128])."""
    H = int(W_UK.shape[0])
    for t in (W_UK, W_UV, R):
        assert t.dtype == torch.float32
    assert tuple(W_UK.shape) == (H, D_C, D_NOPE) and tuple(W_UV.shape) == (H, D_C, D_V)
    assert tuple(R.shape) == (D_C, D_C)
    W_q = torch.empty((H, D_NOPE, D_C), dtype=torch.bfloat16, device=W_UK.device)
    W_o = torch.empty((H, D_C, D_V), dtype=torch.bfloat16, device=W_UK.device)
    _check("rolaq_fold_weights", lib().rolaq_fold_weights(
        _ptr(W_UK), _ptr(W_UV), _ptr(R), H, _ptr(W_q), _ptr(W_o), _stream(stream)))
    return W_q, W_o


def fold_query(q_nope: torch.Tensor, W_q: torch.Tensor, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """rolaq_fold_query: q_nope bf16 [B, H, 128] -> q_c_rot bf16 [B, H, 512]."""
    B, H = int(q_nope.shape[0]), int(q_nope.shape[1])
    assert q_nope.dtype == torch.bfloat16 and tuple(q_nope.shape) == (B, H, D_NOPE)
    assert W_q.dtype == torch.bfloat16 and tuple(W_q.shape) == (H, D_NOPE, D_C)
    if out is None:
        out = torch.empty((B, H, D_C), dtype=torch.bfloat16, device=q_nope.device)
    _check("rolaq_fold_query", lib().rolaq_fold_query(_ptr(q_nope), _ptr(W_q), B, H, _ptr(out),
                                                      _stream(stream)))
    return out


def unfold_output(out_rot: torch.Tensor, W_o: torch.Tensor, v: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """rolaq_unfold_output: out_rot fp32 [B, H, 512] -> v fp32 [B, H, 128]."""
    B, H = int(out_rot.shape[0]), int(out_rot.shape[1])
    assert out_rot.dtype == torch.float32 and tuple(out_rot.shape) == (B, H, D_C)
    assert W_o.dtype == torch.bfloat16 and tuple(W_o.shape) == (H, D_C, D_V)
    if v is None:
        v = torch.empty((B, H, D_V), dtype=torch.float32, device=out_rot.device)
    _check("rolaq_unfold_output", lib().rolaq_unfold_output(_ptr(out_rot), _ptr(W_o), B, H, _ptr(v),
                                                            _stream(stream)))
    return v


def get_status(stream=None) -> int:
    """rolaq_get_status: the device status bits (STATUS_*) since the last read; clears them."""
    v = ctypes.c_int(0)
    _check("rolaq_get_status", lib().rolaq_get_status(ctypes.byref(v), _stream(stream)))
    return v.value
