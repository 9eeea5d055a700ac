"""Thin Python binding over libsafe_attn.so (argument marshalling only).

Every function takes CUDA torch tensors, checks their dtype / shape /
contiguity, passes raw pointers and the current torch stream to the C ABI of
``include/safe_attn.h`` and raises ``SafeError`` on a non-OK status. All
computation runs in the library's CUDA kernels; there is no CPU fallback: if
the library is missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsafe_attn.so")
_lib = None

SAFE_OK, SAFE_ERR_INVALID_ARG, SAFE_ERR_UNSUPPORTED, SAFE_ERR_CUDA, SAFE_ERR_TIMEOUT, SAFE_ERR_DEVICE_CHECK = range(6)
_MASK_DTYPES = {torch.bool: 0, torch.uint8: 1, torch.float32: 2, torch.float16: 3, torch.bfloat16: 4}

_vp, _i, _f, _i64p, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_int64), ctypes.c_size_t

# name -> argtypes (restype is int for every entry point except the ones listed)
_SIGS = {
    "safe_abi_version": [],
    "safe_mask_classify": [_vp, _i, _i64p, _i64p, _vp, _vp],
    "safe_mask_classify_sync": [_vp, _i, _i64p, _i64p, _vp, _i64p, _vp],
    "safe_attn_workspace_bytes": [_i, _i, _i, _i, _i],
    "safe_attn_self": [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz, _vp],
    "safe_attn_cross": [_vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp],
    "safe_pcsp_workspace_bytes": [_i, _i, _i],
    "safe_pcsp_topk": [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _i, _i, _vp, _vp, _vp, _sz, _vp],
    "safe_topk_partition": [_vp, _i, _i, _i, _vp, _vp, _vp],
    "safe_srsu_workspace_bytes": [_i, _i, _i, _i, _i],
    "safe_srsu_attn": [_vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz, _vp],
    "safe_srsu_attn_assembled": [_vp, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz,
                                 _vp],
    "safe_ctx_cache_scatter": [_vp, _vp, _i, _vp, _i, _vp, _vp, _i, _i, _i, _i, _vp],
    "safe_get_device_status": [ctypes.POINTER(ctypes.c_int), _vp],
    "safe_status_string": [_i],
    "safe_selftest_wait_timeout": [ctypes.c_uint64, _vp],
    "safe_pcsp_topk_noalloc": [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _i, _i, _vp, _vp, _vp],
    "safe_attn_cross_pcsp": [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _i, _i, _vp, _vp, _vp,
                             _sz, _vp],
    "safe_sensitivity_workspace_bytes": [_i, _i],
    "safe_sensitivity_field": [_vp, _vp, _i, _i, _i, _f, _f, _vp, _sz, _vp],
    "safe_partition_indicator": [_vp, _i, _vp, _i, _i, _vp],
    "safe_sw_cfg": [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _f, _vp],
    "safe_gather_linear_workspace_bytes": [_i, _i, _i],
    "safe_gather_linear": [_vp, _vp, _i, _vp, _vp, _i, _vp, _i, _i, _i, _i, _vp, _sz, _vp],
}
_RESTYPES = {"safe_pcsp_workspace_bytes": _sz, "safe_attn_workspace_bytes": _sz, "safe_sensitivity_workspace_bytes": _sz,
             "safe_gather_linear_workspace_bytes": _sz, "safe_srsu_workspace_bytes": _sz,
             "safe_status_string": ctypes.c_char_p}


class SafeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({_status_string(status)})")


def lib():
    """Load libsafe_attn.so (once). Raises if it is missing: no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m mask_free_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = _RESTYPES.get(name, ctypes.c_int)
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _status_string(st: int) -> str:
    try:
        return lib().safe_status_string(st).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(fn: str, st: int):
    if st != SAFE_OK:
        raise SafeError(fn, st)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _on_device(t: torch.Tensor) -> bool:
    return t.is_cuda


def _need(t: torch.Tensor, name: str, dtype, ndim: int, shape=None, device=None):
    """Check a tensor argument: a contiguous CUDA tensor of `dtype` and `ndim`
    dims; with `shape` exactly that shape, with `device` on that device. The
    library trusts the sizes it is given, so every tensor whose extent follows
    from another argument is checked here before any launch."""
    if not isinstance(t, torch.Tensor) or not _on_device(t):
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(t, name: str, dtype, shape, device):
    """An output buffer: a new one, or the given one checked like an input."""
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=device)
    _need(t, name, dtype, len(shape), shape, device)
    return t


def _text_kv(Ky, Vy, B, H, d, device):
    """Check the text keys / values [B, M, H, d]; returns M."""
    _need(Ky, "Ky", torch.bfloat16, 4, device=device)
    M = Ky.shape[1]
    _need(Ky, "Ky", torch.bfloat16, 4, (B, M, H, d), device)
    if Vy is not None:
        _need(Vy, "Vy", torch.bfloat16, 4, (B, M, H, d), device)
    return M


def _split_bufs(S, C, B, N, k, device, with_c=True):
    """S [B, k] and C [B, N - k] int32 buffers of the top-k split."""
    if k > N:
        raise ValueError(f"k = {k} exceeds N = {N}")
    S = _out(S, "S", torch.int32, (B, k), device)
    if with_c:
        C = _out(C, "C", torch.int32, (B, N - k), device)
    return S, C


def abi_version() -> int:
    return lib().safe_abi_version()


def mask_classify(mask: torch.Tensor, sync: bool = True, result: Optional[torch.Tensor] = None):
    """Row-constant mask classification (Eq. (6)) of a 4-D [B, H, n_q, n_k]
    mask view (any strides; stride 0 = broadcast). Returns (verdict, nfail,
    first_fail) as Python ints when sync, else the device int64[3] tensor."""
    if not isinstance(mask, torch.Tensor) or mask.dim() != 4 or not _on_device(mask) or mask.dtype not in _MASK_DTYPES:
        raise ValueError("mask must be a 4-D CUDA tensor of dtype bool/uint8/float32/float16/bfloat16")
    sizes = (ctypes.c_int64 * 4)(*mask.shape)
    strides = (ctypes.c_int64 * 4)(*mask.stride())
    result = _out(result, "result", torch.int64, (3,), mask.device)
    if sync:
        h = (ctypes.c_int64 * 3)()
        _check("safe_mask_classify_sync",
               lib().safe_mask_classify_sync(_p(mask), _MASK_DTYPES[mask.dtype], sizes, strides, _p(result), h,
                                             _stream()))
        return int(h[0]), int(h[1]), int(h[2])
    _check("safe_mask_classify",
           lib().safe_mask_classify(_p(mask), _MASK_DTYPES[mask.dtype], sizes, strides, _p(result), _stream()))
    return result


def _scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def attn_workspace_bytes(B: int, n_q: int, N: int, H: int, d: int) -> int:
    return int(lib().safe_attn_workspace_bytes(B, n_q, N, H, d))


def _attn_ws(ws, B, n_q, N, H, d, device):
    """Workspace for the wave-balancing key split: the given tensor, a fresh
    one (ws=None), or no split at all (ws=False)."""
    if ws is False:
        return None, 0
    if ws is None:
        nbytes = attn_workspace_bytes(B, n_q, N, H, d)
        if nbytes == 0:
            return None, 0
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def attn_self(Q, K, V, scale=None, return_lse=False, out=None, lse=None, ws=None):
    """Mask-free image self-attention (Eq. (3) with the mask elided)."""
    _need(Q, "Q", torch.bfloat16, 4)
    B, N, H, d = Q.shape
    dev = Q.device
    _need(K, "K", torch.bfloat16, 4, Q.shape, dev)
    _need(V, "V", torch.bfloat16, 4, Q.shape, dev)
    out = _out(out, "out", torch.bfloat16, (B, N, H, d), dev)
    if return_lse:
        lse = _out(lse, "lse", torch.float32, (B, H, N), dev)
    w, wb = _attn_ws(ws, B, N, N, H, d, Q.device)
    _check("safe_attn_self", lib().safe_attn_self(_p(Q), _p(K), _p(V), _p(out), _p(lse if return_lse else None),
                                                  B, N, H, d, _scale(d, scale), _p(w), wb, _stream()))
    return (out, lse) if return_lse else out


def attn_cross(Q, Ky, Vy, valid_len, q_idx=None, scale=None, out=None):
    """Image->text cross-attention with the padding kept as valid lengths
    (Eq. (4)); with q_idx = S the row-selective form (Eq. (17))."""
    _need(Q, "Q", torch.bfloat16, 4)
    B, N, H, d = Q.shape
    dev = Q.device
    M = _text_kv(Ky, Vy, B, H, d, dev)
    _need(valid_len, "valid_len", torch.int32, 1, (B,), dev)
    nq = N
    if q_idx is not None:
        _need(q_idx, "q_idx", torch.int32, 2, device=dev)
        nq = q_idx.shape[1]
        _need(q_idx, "q_idx", torch.int32, 2, (B, nq), dev)
    out = _out(out, "out", torch.bfloat16, (B, nq, H, d), dev)
    _check("safe_attn_cross", lib().safe_attn_cross(_p(Q), _p(q_idx), nq, _p(Ky), _p(Vy), _p(valid_len), _p(out),
                                                    B, N, M, H, d, _scale(d, scale), _stream()))
    return out


def pcsp_workspace_bytes(B: int, N: int, H: int) -> int:
    return int(lib().safe_pcsp_workspace_bytes(B, N, H))


def pcsp_topk(Q, Ky, valid_len, w=None, scores=None, accumulate=False, k=0, scale=None, S=None, C=None, ws=None):
    """PCSP scores (Eq. (10)) for one step / layer and, if k > 0, the top-k
    partition (Eq. (12)). Returns (scores, S, C)."""
    if Q is not None:
        _need(Q, "Q", torch.bfloat16, 4)
        B, N, H, d = Q.shape
        dev = Q.device
        M = _text_kv(Ky, None, B, H, d, dev)
        _need(valid_len, "valid_len", torch.int32, 1, (B,), dev)
        if w is not None:
            _need(w, "w", torch.float32, 2, (B, M), dev)
    else:
        _need(scores, "scores", torch.float32, 2)
        B, N = scores.shape
        H, d, M = 1, 64, 1
        dev = scores.device
    if scores is None:
        scores = torch.zeros((B, N), dtype=torch.float32, device=dev)
    else:
        _need(scores, "scores", torch.float32, 2, (B, N), dev)
    if k > 0:
        S, C = _split_bufs(S, C, B, N, k, dev)
    nbytes = pcsp_workspace_bytes(B, N, H) if Q is not None else 0
    if Q is not None and ws is None:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check("safe_pcsp_topk", lib().safe_pcsp_topk(
        _p(Q), _p(Ky), _p(valid_len), _p(w), B, N, M, H, d, _scale(d, scale), _p(scores), 1 if accumulate else 0, k,
        _p(S), _p(C), _p(ws), ws.numel() if ws is not None else 0, _stream()))
    return scores, S, C


def attn_cross_pcsp(Q, Ky, Vy, valid_len, w=None, out=None, scores=None, accumulate=False, k=0, scale=None, S=None,
                    C=None, ws=None):
    """Cross-attention (Eq. (4)) and the PCSP scores of Eq. (10) from the same
    probabilities, in one pass over Q; with k > 0 also the top-k split
    (Eq. (12)). Returns (O, scores, S, C)."""
    _need(Q, "Q", torch.bfloat16, 4)
    B, N, H, d = Q.shape
    dev = Q.device
    M = _text_kv(Ky, Vy, B, H, d, dev)
    _need(valid_len, "valid_len", torch.int32, 1, (B,), dev)
    if w is not None:
        _need(w, "w", torch.float32, 2, (B, M), dev)
    out = _out(out, "out", torch.bfloat16, (B, N, H, d), dev)
    if scores is None:
        scores = torch.zeros((B, N), dtype=torch.float32, device=dev)
    else:
        _need(scores, "scores", torch.float32, 2, (B, N), dev)
    if k > 0:
        S, C = _split_bufs(S, C, B, N, k, dev)
    if ws is None:
        ws = torch.empty(max(pcsp_workspace_bytes(B, N, H), 256), dtype=torch.uint8, device=Q.device)
    _check("safe_attn_cross_pcsp", lib().safe_attn_cross_pcsp(
        _p(Q), _p(Ky), _p(Vy), _p(valid_len), _p(w), _p(out), B, N, M, H, d, _scale(d, scale), _p(scores),
        1 if accumulate else 0, k, _p(S), _p(C), _p(ws), ws.numel(), _stream()))
    return out, scores, S, C


def topk_partition(scores, k, S=None, C=None, with_c=True):
    """Exact tie-stable top-k split of Eq. (12) on given scores."""
    _need(scores, "scores", torch.float32, 2)
    B, N = scores.shape
    S, C = _split_bufs(S, C, B, N, k, scores.device, with_c)
    _check("safe_topk_partition", lib().safe_topk_partition(_p(scores), B, N, k, _p(S), _p(C if with_c else None),
                                                            _stream()))
    return S, C


def srsu_workspace_bytes(B: int, k: int, N: int, H: int, d: int) -> int:
    return int(lib().safe_srsu_workspace_bytes(B, k, N, H, d))


def _srsu_ws(ws, B, k, N, H, d, device):
    """Workspace of an SRSU call: the given tensor, a fresh one of
    srsu_workspace_bytes (ws=None: room for the compact query rows and the
    key split), or none (ws=False)."""
    if ws is False:
        return None, 0
    if ws is None:
        nbytes = srsu_workspace_bytes(B, k, N, H, d)
        if nbytes == 0:
            return None, 0
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def _srsu_args(Q, S, Kc, Vc, q_compact):
    """Check the SRSU inputs: cache K/V [B, N, H, d], S [B, k], Q [B, k, H, d]
    (compact) or [B, N, H, d]; returns B, N, H, d, k, device."""
    _need(Kc, "Kc", torch.bfloat16, 4)
    B, N, H, d = Kc.shape
    dev = Kc.device
    _need(Vc, "Vc", torch.bfloat16, 4, Kc.shape, dev)
    _need(S, "S", torch.int32, 2, device=dev)
    k = S.shape[1]
    _need(S, "S", torch.int32, 2, (B, k), dev)
    _need(Q, "Q", torch.bfloat16, 4, (B, k if q_compact else N, H, d), dev)
    return B, N, H, d, k, dev


def srsu_attn(Q, S, Kc, Vc, q_compact=False, scale=None, return_lse=False, out=None, lse=None, ws=None):
    """SRSU selective self-attention (Eq. (16)): rows S of Q against all N
    keys of the assembled global K/V."""
    B, N, H, d, k, dev = _srsu_args(Q, S, Kc, Vc, q_compact)
    out = _out(out, "out", torch.bfloat16, (B, k, H, d), dev)
    if return_lse:
        lse = _out(lse, "lse", torch.float32, (B, H, k), dev)
    w, wb = _srsu_ws(ws, B, k, N, H, d, dev)
    _check("safe_srsu_attn", lib().safe_srsu_attn(_p(Q), 1 if q_compact else 0, _p(S), k, _p(Kc), _p(Vc), _p(out),
                                                  _p(lse if return_lse else None), B, N, H, d, _scale(d, scale),
                                                  _p(w), wb, _stream()))
    return (out, lse) if return_lse else out


def srsu_attn_assembled(Q, S, Kcur, Vcur, Kc, Vc, q_compact=False, cur_compact=False, scale=None, return_lse=False,
                        out=None, lse=None, ws=None):
    """SRSU (Eq. (16)) with K/V of S u C assembled in the kernel (Eq. (14)):
    rows of S from the current Kcur/Vcur ([B, k, H, d] when cur_compact, else
    [B, N, H, d]), the other rows from the cache Kc/Vc, which is not written.
    S must be strictly ascending."""
    B, N, H, d, k, dev = _srsu_args(Q, S, Kc, Vc, q_compact)
    cur_shape = (B, k if cur_compact else N, H, d)
    _need(Kcur, "Kcur", torch.bfloat16, 4, cur_shape, dev)
    _need(Vcur, "Vcur", torch.bfloat16, 4, cur_shape, dev)
    out = _out(out, "out", torch.bfloat16, (B, k, H, d), dev)
    if return_lse:
        lse = _out(lse, "lse", torch.float32, (B, H, k), dev)
    w, wb = _srsu_ws(ws, B, k, N, H, d, dev)
    _check("safe_srsu_attn_assembled", lib().safe_srsu_attn_assembled(
        _p(Q), 1 if q_compact else 0, _p(S), k, _p(Kcur), _p(Vcur), 1 if cur_compact else 0, _p(Kc), _p(Vc), _p(out),
        _p(lse if return_lse else None), B, N, H, d, _scale(d, scale), _p(w), wb, _stream()))
    return (out, lse) if return_lse else out


def ctx_cache_scatter(Ksrc, Vsrc, S, Kc, Vc, src_compact=True):
    """In-place cache update (Eq. (14)/(16)); S=None is the anchor refresh
    (Eq. (19))."""
    _need(Kc, "Kc", torch.bfloat16, 4)
    B, N, H, d = Kc.shape
    dev = Kc.device
    _need(Vc, "Vc", torch.bfloat16, 4, Kc.shape, dev)
    k = 0
    if S is not None:
        _need(S, "S", torch.int32, 2, device=dev)
        k = S.shape[1]
        _need(S, "S", torch.int32, 2, (B, k), dev)
    src_shape = (B, k, H, d) if (src_compact and S is not None) else (B, N, H, d)
    _need(Ksrc, "Ksrc", torch.bfloat16, 4, src_shape, dev)
    _need(Vsrc, "Vsrc", torch.bfloat16, 4, src_shape, dev)
    _check("safe_ctx_cache_scatter", lib().safe_ctx_cache_scatter(
        _p(Ksrc), _p(Vsrc), 1 if (src_compact and S is not None) else 0, _p(S), k, _p(Kc), _p(Vc), B, N, H, d,
        _stream()))
    return Kc, Vc


def device_status() -> int:
    """Read and clear the library's device status word (synchronises)."""
    v = ctypes.c_int(0)
    _check("safe_get_device_status", lib().safe_get_device_status(ctypes.byref(v), _stream()))
    return v.value


def selftest_wait_timeout(limit_ns: int = 1_000_000) -> None:
    """Launch the bounded-wait self-test (see safe_selftest_wait_timeout)."""
    _check("safe_selftest_wait_timeout", lib().safe_selftest_wait_timeout(int(limit_ns), _stream()))


def shared_partition(scores, k, sample: int = 0, B: int = None):
    """One partition for a whole CFG pair (or batch): the top-k split of
    Eq. (12) of one sample's scores (by default the conditional one,
    sample 0), repeated for every sample, so that all of them update the
    same sensitive rows. Returns S [B, k], C [B, N - k] (int32, device)."""
    _need(scores, "scores", torch.float32, 2)
    B = scores.shape[0] if B is None else B
    S1, C1 = topk_partition(scores[sample:sample + 1], k)
    return S1.expand(B, -1).contiguous(), C1.expand(B, -1).contiguous()


def sensitivity_workspace_bytes(B: int, N: int) -> int:
    return int(lib().safe_sensitivity_workspace_bytes(B, N))


def sensitivity_field(scores, grid_h: int, grid_w: int, sigma: float, truncate: float = 4.0, out=None, ws=None):
    """s = Norm(G_sigma * s~) of Eq. (11) on the grid_h x grid_w latent grid
    (row-major tokens), per sample: [B, N] fp32 -> [B, N] fp32 in [0, 1]."""
    _need(scores, "scores", torch.float32, 2)
    B, N = scores.shape
    if N != grid_h * grid_w:
        raise ValueError(f"scores hold {N} tokens per sample, the grid {grid_h} x {grid_w} has {grid_h * grid_w}")
    out = _out(out, "out", torch.float32, (B, N), scores.device)
    nbytes = sensitivity_workspace_bytes(B, N)
    if ws is None:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=scores.device)
    _check("safe_sensitivity_field", lib().safe_sensitivity_field(
        _p(scores), _p(out), B, grid_h, grid_w, float(sigma), float(truncate), _p(ws), ws.numel(), _stream()))
    return out


def partition_indicator(S, N: int, out=None):
    """Binary field of the SW-CFG binary variant: 1 on S, 0 on C ([B, N] fp32)."""
    _need(S, "S", torch.int32, 2)
    B, k = S.shape
    out = _out(out, "out", torch.float32, (B, N), S.device)
    _check("safe_partition_indicator", lib().safe_partition_indicator(_p(S), k, _p(out), B, N, _stream()))
    return out


_CFG_DTYPES = {torch.float32: 2, torch.bfloat16: 4}


def sw_cfg(f_c, f_u, s, gamma_ctx: float, gamma_sens: float, out=None):
    """Sensitivity-weighted CFG, Eq. (20), (21): f_u + gamma_i (f_c - f_u),
    gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) s_i. f_c, f_u [B, N, C]
    (fp32 or bf16), s [B, N] fp32; out may be f_c or f_u (in place)."""
    if f_c.dtype not in _CFG_DTYPES or f_u.dtype != f_c.dtype:
        raise ValueError("f_c and f_u must both be float32 or both bfloat16")
    _need(f_c, "f_c", f_c.dtype, 3)
    B, N, C = f_c.shape
    dev = f_c.device
    _need(f_u, "f_u", f_c.dtype, 3, f_c.shape, dev)
    _need(s, "s", torch.float32, 2, (B, N), dev)
    out = _out(out, "out", f_c.dtype, (B, N, C), dev)
    _check("safe_sw_cfg", lib().safe_sw_cfg(_p(f_c), _p(f_u), _p(s), _p(out), _CFG_DTYPES[f_c.dtype], B, N, C,
                                            float(gamma_ctx), float(gamma_sens), _stream()))
    return out



_ACTS = {"none": 0, "gelu_tanh": 1}


def gather_linear_workspace_bytes(B: int, k: int, d_in: int) -> int:
    return int(lib().safe_gather_linear_workspace_bytes(B, k, d_in))


def gather_linear(X, Wt, S=None, bias=None, act="none", out=None, ws=None):
    """A row-wise layer of the row-selective block (Eq. (13), (15)):
    Y[b, r, :] = act(X[b, S[b, r], :] W^T + bias); S = None: every row (the
    dense block). X [B, N, d_in] bf16, Wt [d_out, d_in] bf16, S [B, k] int32,
    bias [d_out] fp32, act "none" or "gelu_tanh". Returns [B, k or N, d_out].
    ws: the workspace for the compact copy of the rows of S (a fresh one when
    None; False: the GEMM gathers the rows itself)."""
    _need(X, "X", torch.bfloat16, 3)
    B, N, d_in = X.shape
    dev = X.device
    _need(Wt, "Wt", torch.bfloat16, 2, device=dev)
    d_out = Wt.shape[0]
    _need(Wt, "Wt", torch.bfloat16, 2, (d_out, d_in), dev)
    k, R = 0, N
    if S is not None:
        _need(S, "S", torch.int32, 2, device=dev)
        k = R = S.shape[1]
        _need(S, "S", torch.int32, 2, (B, k), dev)
    if bias is not None:
        _need(bias, "bias", torch.float32, 1, (d_out,), dev)
    if act not in _ACTS:
        raise ValueError(f"act must be one of {sorted(_ACTS)}, got {act!r}")
    out = _out(out, "out", torch.bfloat16, (B, R, d_out), dev)
    w, wb = None, 0
    if S is not None and ws is not False:
        if ws is None:
            ws = torch.empty(gather_linear_workspace_bytes(B, k, d_in), dtype=torch.uint8, device=dev)
        _need(ws, "ws", torch.uint8, 1, device=dev)
        w, wb = ws, ws.numel()
    _check("safe_gather_linear", lib().safe_gather_linear(_p(X), _p(S), k, _p(Wt), _p(bias), _ACTS[act], _p(out), B,
                                                          N, d_in, d_out, _p(w), wb, _stream()))
    return out
