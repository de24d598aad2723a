"""Python binding of libb200attn.so: non-causal long-sequence attention on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
library; torch tensors supply device memory and the current stream.  There
is no CPU or eager fallback: if the library is missing or the device is not
an sm_100 part, calls raise.

Tensor layouts (batch 1):
  q, k, v, out  fp16 [S, H, d]; rows may be strided (views into a fused QKV
                buffer), the head and feature dims must be dense.
  lse           fp32 [H, S], natural log of sum_j exp(scale * q.k_j).
  o_parts       fp32 [P, S, H, d];  lse_parts fp32 [P, H, S].
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

# ATTN_DEBUG=1 selects the debug build (every TMA box and TMEM access
# bounds-checked on the device before it is issued; same entry points).
_DEBUG = os.environ.get("ATTN_DEBUG", "0") not in ("", "0")
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                         "libb200attn_debug.so" if _DEBUG else "libb200attn.so")

__all__ = [
    "B2AError", "lib", "attn_fwd", "attn_fwd_batched", "attn_fwd_gathered_kv", "attn_fwd_partial", "attn_fwd_accumulate",
    "attn_fwd_partial_f16", "attn_fwd_partials", "attn_merge", "attn_merge_f16", "attn_chunked", "attn_ring", "set_attn_kernel", "get_attn_kernel", "attn_kernel_for",
    "ATTN_KERNEL_AUTO", "ATTN_KERNEL_SINGLE", "ATTN_KERNEL_PAIR",
    "qkv_proj", "qkv_proj_qknorm", "out_proj", "attn_block_fwd", "stack_forward", "attn_fwd_host",
    "host_workspace_bytes", "check_status", "selftest_wait_timeout",
    "chunk_bounds", "library_path",
]

B2A_OK, B2A_ERR_INVALID_ARG, B2A_ERR_UNSUPPORTED, B2A_ERR_CUDA, B2A_ERR_TIMEOUT, B2A_ERR_DEVICE_CHECK = range(6)
ATTN_KERNEL_AUTO, ATTN_KERNEL_SINGLE, ATTN_KERNEL_PAIR = range(3)

_u16p = ctypes.c_void_p
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

_SIGS = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _i, _i, _i, _vp]),
    "attn_fwd_batched": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]),
    "attn_fwd_gathered_kv": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _i, _i, _vp]),
    "attn_fwd_partial": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_accumulate": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "b2a_set_attn_kernel": (_i, [_i]),
    "b2a_get_attn_kernel": (_i, []),
    "b2a_attn_kernel_for": (_i, [_i, _i]),
    "attn_merge": (_i, [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _vp]),
    "attn_fwd_partial_f16": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_merge_f16": (_i, [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _vp]),
    "attn_fwd_partials": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_partials_f16": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "qkv_proj": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "attn_block_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp]),
    "attn_block_fwd_static": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp]),
    "out_proj": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "qkv_proj_qknorm": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]),
    "attn_block_fwd_qknorm": (_i, [_vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp]),
    "attn_fwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp, ctypes.c_uint64, _vp]),
    "attn_fwd_host_workspace_bytes": (ctypes.c_uint64, [_i, _i, _i, _i]),
    "b2a_check_status": (_i, [_vp]),
    "b2a_selftest_wait_timeout": (_i, [_i, _vp, _vp]),
    "b2a_status_string": (ctypes.c_char_p, [_i]),
    "b2a_last_cuda_error": (_i, []),
    "b2a_version": (_i, []),
    "b2a_debug_build": (_i, []),
}


class B2AError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        lib_ = _get_lib()
        msg = lib_.b2a_status_string(status).decode()
        extra = ""
        if status == B2A_ERR_CUDA:
            extra = f" (cudaError {lib_.b2a_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}{extra}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libb200attn.so not found at {_LIB_PATH}; build it with "
            "`python -m long_context_bidirectional_b200.build` (needs nvcc)")
    handle = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


_lib = None


def _get_lib() -> ctypes.CDLL:
    """Load libb200attn.so on first use; raises ImportError if it is missing."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def __getattr__(name):
    if name == "lib":
        return _get_lib()
    raise AttributeError(name)


def library_path() -> str:
    return _LIB_PATH


def _call(name: str, *args) -> None:
    st = getattr(_get_lib(), name)(*args)
    if st != B2A_OK:
        raise B2AError(name, st)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_qkv(name: str, t: torch.Tensor, H: int | None = None, d: int | None = None) -> int:
    """Validate an fp16 CUDA [S, H, d] view; return its row stride in elements."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.float16:
        raise TypeError(f"{name} must be float16, got {t.dtype}")
    if t.dim() != 3:
        raise ValueError(f"{name} must be [S, H, d], got shape {tuple(t.shape)}")
    S_, H_, d_ = t.shape
    if (H is not None and H_ != H) or (d is not None and d_ != d):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected [*, {H}, {d}]")
    if t.stride(2) != 1 or (H_ > 1 and t.stride(1) != d_):
        raise ValueError(f"{name}: head and feature dims must be dense (strides {t.stride()})")
    return t.stride(0) if S_ > 1 else max(t.stride(0), H_ * d_)


def _default_scale(d: int, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def attn_fwd(q, k, v, out=None, lse=None, scale=None, return_lse=True, stream=None):
    """Monolithic non-causal attention; returns ``(out, lse)`` (lse may be None)."""
    S, H, d = q.shape
    ld_q = _check_qkv("q", q)
    ld_k = _check_qkv("k", k, H, d)
    ld_v = _check_qkv("v", v, H, d)
    if k.shape[0] != S or v.shape[0] != S:
        raise ValueError("attn_fwd is self-attention: q, k, v need the same S")
    if out is None:
        out = torch.empty((S, H, d), dtype=torch.float16, device=q.device)
    ld_o = _check_qkv("out", out, H, d)
    if lse is None and return_lse:
        lse = torch.empty((H, S), dtype=torch.float32, device=q.device)
    _call("attn_fwd", q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
          S, H, d, _default_scale(d, scale), ld_q, ld_k, ld_v, ld_o, _stream(stream))
    return out, lse


def attn_fwd_batched(q, k, v, out=None, lse=None, scale=None, return_lse=True, stream=None):
    """attn_fwd over ``[S, B, H, d]`` contiguous tensors (the (S, B, hidden)
    layout); returns ``(out [S,B,H,d], lse [B,H,S])``."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.float16):
            raise TypeError(f"{name} must be a float16 CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError(f"{name} must be contiguous [S, B, H, d] like q")
    S, B, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if not (out.is_contiguous() and out.shape == q.shape and out.dtype == torch.float16):
        raise ValueError("out must be contiguous float16 [S, B, H, d]")
    if lse is None and return_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _call("attn_fwd_batched", q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
          S, B, H, d, _default_scale(d, scale), _stream(stream))
    return out, lse


def attn_fwd_gathered_kv(q, k, v, out=None, lse=None, scale=None, return_lse=True, stream=None):
    """One AllGather-KV context-parallel rank: its ``q [Sq,H,d]`` rows against
    all ``k, v [Skv,H,d]``; returns ``(out [Sq,H,d] fp16, lse [H,Sq])``."""
    Sq, H, d = q.shape
    ld_q = _check_qkv("q", q)
    ld_k = _check_qkv("k", k, H, d)
    ld_v = _check_qkv("v", v, H, d)
    Skv = k.shape[0]
    if v.shape[0] != Skv:
        raise ValueError("k and v need the same length")
    if out is None:
        out = torch.empty((Sq, H, d), dtype=torch.float16, device=q.device)
    ld_o = _check_qkv("out", out, H, d)
    if lse is None and return_lse:
        lse = torch.empty((H, Sq), dtype=torch.float32, device=q.device)
    _call("attn_fwd_gathered_kv", q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
          Sq, Skv, H, d, _default_scale(d, scale), ld_q, ld_k, ld_v, ld_o, _stream(stream))
    return out, lse


def attn_fwd_partial(q, k_chunk, v_chunk, o_part=None, lse_part=None, scale=None, stream=None):
    """Attention of all queries against one key chunk; returns ``(o_part, lse_part)``."""
    return _partial("attn_fwd_partial", torch.float32, q, k_chunk, v_chunk, o_part, lse_part, scale, stream)


def attn_fwd_partial_f16(q, k_chunk, v_chunk, o_part=None, lse_part=None, scale=None, stream=None):
    """``attn_fwd_partial`` with ``o_part`` stored in fp16 (the FP16 split-reduction)."""
    return _partial("attn_fwd_partial_f16", torch.float16, q, k_chunk, v_chunk, o_part, lse_part, scale, stream)


def attn_fwd_partials(q, k, v, P: int, o_parts=None, lse_parts=None, scale=None, stream=None,
                      partial_dtype=torch.float32):
    """Every key chunk's partial in one call: ``(o_parts [P,Sq,H,d], lse_parts [P,H,Sq])``,
    chunk c = keys ``chunk_bounds(Skv, P)[c]`` (fp32 or fp16 ``o_parts``)."""
    Sq, H, d = q.shape
    ld_q = _check_qkv("q", q)
    Skv = k.shape[0]
    ld_k = _check_qkv("k", k, H, d)
    ld_v = _check_qkv("v", v, H, d)
    if v.shape[0] != Skv:
        raise ValueError("k and v need the same length")
    if ld_k != ld_v:
        raise ValueError("k and v must share a row stride")
    if partial_dtype not in (torch.float32, torch.float16):
        raise ValueError("partial_dtype must be torch.float32 or torch.float16")
    if o_parts is None:
        o_parts = torch.empty((P, Sq, H, d), dtype=partial_dtype, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty((P, H, Sq), dtype=torch.float32, device=q.device)
    if not (o_parts.is_contiguous() and o_parts.dtype == partial_dtype and o_parts.numel() == P * Sq * H * d):
        raise ValueError(f"o_parts must be contiguous {partial_dtype} [P, Sq, H, d]")
    if not (lse_parts.is_contiguous() and lse_parts.dtype == torch.float32 and lse_parts.numel() == P * H * Sq):
        raise ValueError("lse_parts must be contiguous float32 [P, H, Sq]")
    fn = "attn_fwd_partials_f16" if partial_dtype == torch.float16 else "attn_fwd_partials"
    kp = k.data_ptr() if Skv > 0 else q.data_ptr()
    vp = v.data_ptr() if Skv > 0 else q.data_ptr()
    _call(fn, q.data_ptr(), kp, vp, o_parts.data_ptr(), lse_parts.data_ptr(), Sq, Skv, int(P), H, d,
          _default_scale(d, scale), ld_q, ld_k if Skv > 0 else ld_q, _stream(stream))
    return o_parts, lse_parts


def _partial(fn, odt, q, k_chunk, v_chunk, o_part, lse_part, scale, stream):
    Sq, H, d = q.shape
    ld_q = _check_qkv("q", q)
    Skv = k_chunk.shape[0]
    ld_k = _check_qkv("k_chunk", k_chunk, H, d)
    ld_v = _check_qkv("v_chunk", v_chunk, H, d)
    if v_chunk.shape[0] != Skv:
        raise ValueError("k_chunk and v_chunk need the same length")
    if ld_k != ld_v:
        raise ValueError("k_chunk and v_chunk must share a row stride")
    if o_part is None:
        o_part = torch.empty((Sq, H, d), dtype=odt, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((H, Sq), dtype=torch.float32, device=q.device)
    if not (o_part.is_contiguous() and o_part.dtype == odt and o_part.numel() == Sq * H * d):
        raise ValueError(f"o_part must be contiguous {odt} [Sq, H, d]")
    if not (lse_part.is_contiguous() and lse_part.dtype == torch.float32 and lse_part.numel() == H * Sq):
        raise ValueError("lse_part must be contiguous float32 [H, Sq]")
    # An empty chunk may be a zero-length view; any valid address will do.
    kp = k_chunk.data_ptr() if Skv > 0 else q.data_ptr()
    vp = v_chunk.data_ptr() if Skv > 0 else q.data_ptr()
    _call(fn, q.data_ptr(), kp, vp, o_part.data_ptr(), lse_part.data_ptr(),
          Sq, Skv, H, d, _default_scale(d, scale), ld_q, ld_k if Skv > 0 else ld_q, _stream(stream))
    return o_part, lse_part


def attn_fwd_accumulate(q, k_chunk, v_chunk, o_acc, lse_acc, out=None, scale=None, stream=None):
    """One ring step in place: fold a key chunk into ``(o_acc [Sq,H,d] fp32, lse_acc [H,Sq])``.

    ``lse_acc = -inf`` marks rows with no keys yet.  ``out`` (fp16, optional)
    also receives the rounded merged output.  Returns ``(o_acc, lse_acc, out)``.
    """
    Sq, H, d = q.shape
    ld_q = _check_qkv("q", q)
    Skv = k_chunk.shape[0]
    ld_k = _check_qkv("k_chunk", k_chunk, H, d)
    ld_v = _check_qkv("v_chunk", v_chunk, H, d)
    if v_chunk.shape[0] != Skv:
        raise ValueError("k_chunk and v_chunk need the same length")
    if ld_k != ld_v:
        raise ValueError("k_chunk and v_chunk must share a row stride")
    if not (o_acc.is_contiguous() and o_acc.dtype == torch.float32 and o_acc.numel() == Sq * H * d):
        raise ValueError("o_acc must be contiguous float32 [Sq, H, d]")
    if not (lse_acc.is_contiguous() and lse_acc.dtype == torch.float32 and lse_acc.numel() == H * Sq):
        raise ValueError("lse_acc must be contiguous float32 [H, Sq]")
    if out is not None and not (out.is_contiguous() and out.dtype == torch.float16
                                and out.numel() == Sq * H * d):
        raise ValueError("out must be contiguous float16 [Sq, H, d]")
    kp = k_chunk.data_ptr() if Skv > 0 else q.data_ptr()
    vp = v_chunk.data_ptr() if Skv > 0 else q.data_ptr()
    _call("attn_fwd_accumulate", q.data_ptr(), kp, vp, o_acc.data_ptr(), lse_acc.data_ptr(), _ptr(out),
          Sq, Skv, H, d, _default_scale(d, scale), ld_q, ld_k if Skv > 0 else ld_q, _stream(stream))
    return o_acc, lse_acc, out


def attn_ring(q, k, v, P: int, out=None, scale=None, o_acc=None, lse_acc=None, stream=None):
    """Ring attention's per-rank loop on one device: P accumulate steps over
    the key chunks, the last one writing the fp16 output.  Returns ``(out, lse_acc)``.
    """
    S, H, d = q.shape
    if o_acc is None:
        o_acc = torch.empty((S, H, d), dtype=torch.float32, device=q.device)
    if lse_acc is None:
        lse_acc = torch.empty((H, S), dtype=torch.float32, device=q.device)
    lse_acc.fill_(float("-inf"))
    if out is None:
        out = torch.empty((S, H, d), dtype=torch.float16, device=q.device)
    bounds = chunk_bounds(k.shape[0], P)
    for c, (lo, hi) in enumerate(bounds):
        attn_fwd_accumulate(q, k[lo:hi], v[lo:hi], o_acc, lse_acc, out if c == P - 1 else None,
                            scale=scale, stream=stream)
    return out, lse_acc


def set_attn_kernel(choice: int) -> None:
    """Head-dim-128 kernel choice: ATTN_KERNEL_AUTO / _SINGLE / _PAIR (process-wide)."""
    _call("b2a_set_attn_kernel", int(choice))


def get_attn_kernel() -> int:
    return int(_get_lib().b2a_get_attn_kernel())


def attn_kernel_for(d: int, Skv: int) -> int:
    """ATTN_KERNEL_SINGLE or ATTN_KERNEL_PAIR: what a call with these sizes uses now."""
    return int(_get_lib().b2a_attn_kernel_for(int(d), int(Skv)))


def attn_merge(o_parts, lse_parts, out=None, lse_out=None, return_lse=True, stream=None):
    """Exact merge of partials ``o_parts [P,S,H,d]`` (fp32), ``lse_parts [P,H,S]``."""
    return _merge("attn_merge", torch.float32, o_parts, lse_parts, out, lse_out, return_lse, stream)


def attn_merge_f16(o_parts, lse_parts, out=None, lse_out=None, return_lse=True, stream=None):
    """``attn_merge`` over fp16 partials (``attn_fwd_partial_f16``'s output)."""
    return _merge("attn_merge_f16", torch.float16, o_parts, lse_parts, out, lse_out, return_lse, stream)


def _merge(fn, odt, o_parts, lse_parts, out, lse_out, return_lse, stream):
    if o_parts.dtype != odt or lse_parts.dtype != torch.float32:
        raise TypeError(f"o_parts must be {odt} and lse_parts float32")
    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("o_parts and lse_parts must be contiguous")
    P, S, H, d = o_parts.shape
    if tuple(lse_parts.shape) != (P, H, S):
        raise ValueError(f"lse_parts must be [P, H, S] = {(P, H, S)}, got {tuple(lse_parts.shape)}")
    if out is None:
        out = torch.empty((S, H, d), dtype=torch.float16, device=o_parts.device)
    if not (out.is_contiguous() and out.dtype == torch.float16 and out.numel() == S * H * d):
        raise ValueError("out must be contiguous float16 [S, H, d]")
    if lse_out is None and return_lse:
        lse_out = torch.empty((H, S), dtype=torch.float32, device=o_parts.device)
    _call(fn, o_parts.data_ptr(), lse_parts.data_ptr(), P, out.data_ptr(), _ptr(lse_out),
          S, H, d, _stream(stream))
    return out, lse_out


def chunk_bounds(S: int, P: int):
    """Chunk ``p`` of ``P`` covers keys ``[floor(p*S/P), floor((p+1)*S/P))``."""
    return [((p * S) // P, ((p + 1) * S) // P) for p in range(P)]


def attn_chunked(q, k, v, P: int, out=None, lse=None, scale=None, o_parts=None, lse_parts=None,
                 stream=None, partial_dtype=torch.float32):
    """Ring attention emulated on one device: P key-chunk partials, then the merge.

    ``partial_dtype`` float32 (default) or float16 (the FP16 split-reduction:
    ``attn_fwd_partial_f16`` + ``attn_merge_f16``).  ``o_parts``/``lse_parts``
    are the caller's workspace (allocated here when omitted).  Returns ``(out, lse)``.
    """
    S, H, d = q.shape
    if partial_dtype not in (torch.float32, torch.float16):
        raise ValueError("partial_dtype must be torch.float32 or torch.float16")
    f16 = partial_dtype == torch.float16
    if o_parts is None:
        o_parts = torch.empty((P, S, H, d), dtype=partial_dtype, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty((P, H, S), dtype=torch.float32, device=q.device)
    attn_fwd_partials(q, k, v, P, o_parts, lse_parts, scale=scale, stream=stream, partial_dtype=partial_dtype)
    merge = attn_merge_f16 if f16 else attn_merge
    return merge(o_parts, lse_parts, out=out, lse_out=lse, stream=stream)


def _check_mat(name, t, rows=None, cols=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float16:
        raise TypeError(f"{name} must be a float16 CUDA tensor")
    if t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")
    if (rows is not None and t.shape[0] != rows) or (cols is not None and t.shape[1] != cols):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected ({rows}, {cols})")


def qkv_proj(x, w_qkv, out=None, stream=None):
    """``out = x @ w_qkv.T``; x [M, K], w_qkv [N, K] fp16."""
    M, K = x.shape
    N = w_qkv.shape[0]
    _check_mat("x", x)
    _check_mat("w_qkv", w_qkv, N, K)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check_mat("out", out, M, N)
    _call("qkv_proj", x.data_ptr(), w_qkv.data_ptr(), out.data_ptr(), M, N, K, _stream(stream))
    return out


def qkv_proj_qknorm(x, w_qkv, g_q, g_k, H: int, d: int, eps: float = 1e-6, out=None, stream=None):
    """``out = x @ w_qkv.T`` with every q and k head RMS-normalised and scaled
    by ``g_q`` / ``g_k`` ([d] fp16) in the GEMM epilogue; v as projected."""
    M, K = x.shape
    N = 3 * H * d
    _check_mat("x", x)
    _check_mat("w_qkv", w_qkv, N, K)
    for name, g in (("g_q", g_q), ("g_k", g_k)):
        if not (isinstance(g, torch.Tensor) and g.is_cuda and g.dtype == torch.float16
                and g.is_contiguous() and g.numel() == d):
            raise ValueError(f"{name} must be a contiguous float16 CUDA tensor of {d} elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check_mat("out", out, M, N)
    _call("qkv_proj_qknorm", x.data_ptr(), w_qkv.data_ptr(), g_q.data_ptr(), g_k.data_ptr(), out.data_ptr(),
          M, H, d, K, float(eps), _stream(stream))
    return out


def out_proj(a, w_o, residual=None, out=None, stream=None):
    """``out = residual + a @ w_o.T`` (residual optional, may be ``out``)."""
    M, K = a.shape
    N = w_o.shape[0]
    _check_mat("a", a)
    _check_mat("w_o", w_o, N, K)
    if residual is not None:
        _check_mat("residual", residual, M, N)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    _check_mat("out", out, M, N)
    _call("out_proj", a.data_ptr(), w_o.data_ptr(), _ptr(residual), out.data_ptr(), M, N, K,
          _stream(stream))
    return out


def attn_block_fwd(x, w_qkv, w_o, H: int, d: int, out=None, qkv_ws=None, attn_ws=None, scale=None,
                   stream=None, qknorm=None):
    """One block: ``out = x + attention(split(x @ w_qkv.T)) @ w_o.T``; ``out`` may be ``x``.

    ``qknorm = (g_q, g_k, eps)`` runs the projection with the q/k RMSNorm
    (``attn_block_fwd_qknorm``).
    """
    S, h = x.shape
    if h != H * d:
        raise ValueError(f"x has {h} columns, expected H*d = {H * d}")
    _check_mat("x", x)
    _check_mat("w_qkv", w_qkv, 3 * h, h)
    _check_mat("w_o", w_o, h, h)
    if out is None:
        out = torch.empty_like(x)
    _check_mat("out", out, S, h)
    if qkv_ws is None:
        qkv_ws = torch.empty((S, 3 * h), dtype=torch.float16, device=x.device)
    if attn_ws is None:
        attn_ws = torch.empty((S, h), dtype=torch.float16, device=x.device)
    _check_mat("qkv_ws", qkv_ws, S, 3 * h)
    _check_mat("attn_ws", attn_ws, S, h)
    if qknorm is None:
        _call("attn_block_fwd", x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), out.data_ptr(),
              qkv_ws.data_ptr(), attn_ws.data_ptr(), S, H, d, _default_scale(d, scale), _stream(stream))
        return out
    g_q, g_k, eps = qknorm
    for name, g in (("g_q", g_q), ("g_k", g_k)):
        if not (isinstance(g, torch.Tensor) and g.is_cuda and g.dtype == torch.float16
                and g.is_contiguous() and g.numel() == d):
            raise ValueError(f"{name} must be a contiguous float16 CUDA tensor of {d} elements")
    _call("attn_block_fwd_qknorm", x.data_ptr(), w_qkv.data_ptr(), g_q.data_ptr(), g_k.data_ptr(), float(eps),
          w_o.data_ptr(), out.data_ptr(), qkv_ws.data_ptr(), attn_ws.data_ptr(), S, H, d,
          _default_scale(d, scale), _stream(stream))
    return out


def stack_forward(x, weights, H: int, d: int, scale=None, stream=None, keep=False):
    """Apply the blocks ``weights = [(w_qkv, w_o), ...]`` in order.

    Returns the final activations, or with ``keep=True`` the list of
    per-block ``(y, qkv, attn)`` (copies of the workspaces after each block).
    """
    S, h = x.shape
    qkv_ws = torch.empty((S, 3 * h), dtype=torch.float16, device=x.device)
    attn_ws = torch.empty((S, h), dtype=torch.float16, device=x.device)
    cur = x.clone()
    kept = []
    for w_qkv, w_o in weights:
        attn_block_fwd(cur, w_qkv, w_o, H, d, out=cur, qkv_ws=qkv_ws, attn_ws=attn_ws, scale=scale,
                       stream=stream)
        if keep:
            kept.append((cur.clone(), qkv_ws.clone(), attn_ws.clone()))
    return kept if keep else cur


def host_workspace_bytes(S: int, H: int, d: int, P: int) -> int:
    return int(_get_lib().attn_fwd_host_workspace_bytes(S, H, d, P))


def attn_fwd_host(q, k, v, out, lse, workspace, P: int = 1, scale=None, stream=None):
    """End-to-end call from host memory (pinned CPU tensors), see the C header."""
    S, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous() or tuple(t.shape) != (S, H, d):
            raise ValueError(f"{name} must be a contiguous float16 host tensor [S, H, d]")
    if lse is not None and (lse.is_cuda or lse.dtype != torch.float32 or lse.numel() != H * S):
        raise ValueError("lse must be a float32 host tensor [H, S]")
    if not workspace.is_cuda:
        raise ValueError("workspace must be device memory")
    _call("attn_fwd_host", q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
          S, H, d, _default_scale(d, scale), P, workspace.data_ptr(),
          workspace.numel() * workspace.element_size(), _stream(stream))
    return out, lse


def check_status(stream=None) -> None:
    """Synchronise and raise if any kernel reported a device-side timeout."""
    _call("b2a_check_status", _stream(stream))


def selftest_wait_timeout(limit_ms: int = 50, stream=None):
    """Run the failure-path self test; returns the device ``result`` tensor.

    Afterwards :func:`check_status` raises once with B2A_ERR_TIMEOUT (and
    clears the status).  See ``b2a_selftest_wait_timeout`` in the C header.
    """
    result = torch.zeros(2, dtype=torch.int32, device="cuda")
    _call("b2a_selftest_wait_timeout", int(limit_ms), result.data_ptr(), _stream(stream))
    return result
