"""Thin Python binding of libcoda.so (the C ABI declared in include/coda.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no fallback:
if the shared library is missing or the device is not a B200, the calls raise.

Names follow the C ABI without the ``coda_`` prefix.  bf16 tensors are passed
as their bit patterns (the C ABI takes ``uint16_t*``), fp32 as ``float*``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcoda.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "coda.h")

CODA_OK = 0
STATUS_NAMES = {
    0: "CODA_OK", 1: "CODA_ERR_NULL", 2: "CODA_ERR_SHAPE", 3: "CODA_ERR_ALIGN",
    4: "CODA_ERR_WORKSPACE", 5: "CODA_ERR_DEVICE", 6: "CODA_ERR_LAUNCH",
    7: "CODA_ERR_DEVICE_TIMEOUT", 8: "CODA_ERR_INTERNAL",
}


class CodaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_ST = ctypes.c_int

_SIGS = {
    "coda_status_string": (ctypes.c_char_p, [_ST]),
    "coda_version": (ctypes.c_int, []),
    "coda_partial_tile_width": (_I64, []),
    "coda_partial_cols": (_I64, [_I64]),
    "coda_set_wait_limit_ns": (_ST, [_I64]),
    "coda_poll_status": (_ST, [_P]),
    "coda_gemm_res_partialrms": (_ST, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_rms_reduce": (_ST, [_P, _I64, _I64, _I64, _F, _P, _P]),
    "coda_gemm_rowscale": (_ST, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_rowscale_partial": (_ST, [_P, _P, _P, _I64, _I64, _F, _P, _P, _I64, _I64, _I64, _P]),
    "coda_rmsnorm_block_workspace_size": (_SZ, [_I64]),
    "coda_rmsnorm_block": (_ST, [_P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _SZ, _I64, _I64, _I64, _I64, _P]),
    "coda_gemm_swiglu": (_ST, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_qkv_rope": (_ST, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _F, _P]),
    "coda_gemm_swiglu_bwd": (_ST, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_lmhead_ce_workspace_size": (_SZ, [_I64, _I64]),
    "coda_lmhead_ce": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _SZ, _I64, _I64, _I64, _P]),
    "coda_lmhead_ce_bwd_workspace_size": (_SZ, [_I64, _I64]),
    "coda_lmhead_ce_bwd": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _I64, _I64, _I64, _P]),
    "coda_loss_stats": (_ST, [_P, _I64, _P, _P]),
    "coda_ce_global_finish": (_ST, [_P, _I64, _P, _P, _P]),
    "coda_gemm_rowscale_bwd_workspace_size": (_SZ, [_I64, _I64]),
    "coda_gemm_rowscale_bwd": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _SZ, _I64, _I64, _I64, _P]),
    "coda_rms_reduce_bwd_workspace_size": (_SZ, [_I64, _I64]),
    "coda_rms_reduce_bwd": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _SZ, _I64, _I64, _I64, _P]),
    "coda_rms_reduce_bwd_noalloc": (_ST, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_res_partialrms_bwd": (_ST, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_unfused_add": (_ST, [_P, _P, _P, _I64, _P]),
    "coda_unfused_rmsnorm": (_ST, [_P, _P, _F, _P, _P, _I64, _I64, _P]),
    "coda_selftest_bounded_wait": (_ST, [_I64, _P, _P]),
    "coda_fp8_quantize": (_ST, [_P, _I64, _I64, ctypes.c_int, _P, _P, _P, _P]),
    "coda_fp8_scale_from_amax": (_ST, [_P, _P, _P]),
    "coda_gemm_res_partialrms_fp8": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_rowscale_partial_fp8": (_ST, [_P, _P, _P, _P, _P, _I64, _I64, _F, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_fp8": (_ST, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_rmsnorm_block_host_workspace_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "coda_rmsnorm_block_host": (_ST, [_P, _P, _P, _P, _P, _F, _P, _P, _SZ, _I64, _I64, _I64, _I64, _I64, _P]),
    "coda_unfused_rmsnorm_fp8": (_ST, [_P, _P, _F, _P, _P, _P, _P, _I64, _I64, _P]),
    "coda_mx_sf_bytes": (_I64, [_I64, _I64, ctypes.c_int]),
    "coda_mx_quantize": (_ST, [_P, _I64, _I64, ctypes.c_int, _P, _P, _P]),
    "coda_gemm_res_partialrms_mx": (_ST, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "coda_gemm_rowscale_partial_mx": (_ST, [_P, _P, _P, _P, _P, _I64, _I64, _F, _P, _P, _I64, _I64, _I64, _P]),
}

_lib = None


def load_library() -> ctypes.CDLL:
    """Load libcoda.so from the package directory (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libcoda.so not found at {LIB_PATH}; build it with "
            "`python -m gemm_epilogue_transformer_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != CODA_OK:
        lib = load_library()
        raise CodaError(fn, status, lib.coda_status_string(status).decode())


# NVTX ranges around every library call (names as in the C ABI), so that a
# timeline profiler shows which call launched which kernels; CODA_NVTX=0
# turns them off.
_NVTX = os.environ.get("CODA_NVTX", "1") != "0"


def _call(name: str, *args):
    lib = load_library()
    if _NVTX:
        torch.cuda.nvtx.range_push(name)
        try:
            st = getattr(lib, name)(*args)
        finally:
            torch.cuda.nvtx.range_pop()
    else:
        st = getattr(lib, name)(*args)
    _check(name, st)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


BF16 = torch.bfloat16
F32 = torch.float32

# ------------------------------------------------------------------ basics


def version() -> int:
    return load_library().coda_version()


def partial_tile_width() -> int:
    return int(load_library().coda_partial_tile_width())


def partial_cols(N: int) -> int:
    return int(load_library().coda_partial_cols(N))


def set_wait_limit_ns(ns: int):
    _call("coda_set_wait_limit_ns", int(ns))


def poll_status():
    """Synchronise the current stream and raise if a kernel recorded a timeout."""
    _call("coda_poll_status", _stream())


# ----------------------------------------------------------------- forward


def gemm_res_partialrms(x, W, res=None, gamma=None, *, h=True, hg=True, partial=True,
                        h_out=None, hg_out=None, partial_out=None):
    """h = x W + res; hg = gamma * h; partial[t, i] = sum_{j in tile t} h_ij^2.
    Returns (h, hg, partial); entries not requested are None."""
    M, K = x.shape
    N = W.shape[1]
    _need(x, BF16, "x")
    _need(W, BF16, "W", (K, N))
    if res is not None:
        _need(res, BF16, "res", (M, N))
    if gamma is not None:
        _need(gamma, BF16, "gamma", (N,))
    if h and h_out is None:
        h_out = _empty((M, N), BF16, x)
    if hg and hg_out is None:
        hg_out = _empty((M, N), BF16, x)
    if partial and partial_out is None:
        partial_out = _empty((partial_cols(N), M), F32, x)
    _call("coda_gemm_res_partialrms", _ptr(x), _ptr(W), _ptr(res), _ptr(gamma),
          _ptr(h_out if h else None), _ptr(hg_out if hg else None),
          _ptr(partial_out if partial else None), M, N, K, _stream())
    return (h_out if h else None, hg_out if hg else None, partial_out if partial else None)


def rms_reduce(partial, N: int, eps: float, r_out=None):
    """r_i = 1 / sqrt(sum_t partial[t, i] / N + eps)."""
    T, M = partial.shape
    _need(partial, F32, "partial")
    if r_out is None:
        r_out = _empty((M,), F32, partial)
    _call("coda_rms_reduce", _ptr(partial), M, T, N, float(eps), _ptr(r_out), _stream())
    return r_out


def gemm_rowscale(A, W, r=None, out=None):
    """out = bf16(r * (A W)); r None gives a plain bf16 GEMM."""
    M, K = A.shape
    N = W.shape[1]
    _need(A, BF16, "A")
    _need(W, BF16, "W", (K, N))
    if r is not None:
        _need(r, F32, "r", (M,))
    if out is None:
        out = _empty((M, N), BF16, A)
    _call("coda_gemm_rowscale", _ptr(A), _ptr(W), _ptr(r), _ptr(out), M, N, K, _stream())
    return out


def gemm_rowscale_partial(A, W, partial, N_norm: int, eps: float, out=None, r_out=None):
    """out = bf16(r * (A W)) with r = 1/sqrt(sum_t partial[t] / N_norm + eps)
    formed in the epilogue; returns (out, r)."""
    M, K = A.shape
    N = W.shape[1]
    T = partial.shape[0]
    _need(A, BF16, "A")
    _need(W, BF16, "W", (K, N))
    _need(partial, F32, "partial", (T, M))
    if out is None:
        out = _empty((M, N), BF16, A)
    if r_out is None:
        r_out = _empty((M,), F32, A)
    _call("coda_gemm_rowscale_partial", _ptr(A), _ptr(W), _ptr(partial), T, int(N_norm), float(eps), _ptr(r_out),
          _ptr(out), M, N, K, _stream())
    return out, r_out


def gemm_swiglu(A, W_gu, r=None, save=False, act_out=None, gateup_out=None):
    """act = silu(r * A W_g) * (r * A W_u); returns (act, gateup or None).
    With save (or gateup_out given) the bf16 gate and up are kept for the backward."""
    M, K = A.shape
    F = W_gu.shape[1] // 2
    _need(A, BF16, "A")
    _need(W_gu, BF16, "W_gu", (K, 2 * F))
    if r is not None:
        _need(r, F32, "r", (M,))
    if act_out is None:
        act_out = _empty((M, F), BF16, A)
    gu = gateup_out
    if gu is not None:
        _need(gu, BF16, "gateup_out", (M, 2 * F))
    elif save:
        gu = _empty((M, 2 * F), BF16, A)
    _call("coda_gemm_swiglu", _ptr(A), _ptr(W_gu), _ptr(r), _ptr(act_out), _ptr(gu), M, F, K, _stream())
    return act_out, gu


def gemm_qkv_rope(x, W_qkv, positions, head_dim: int, rope_cols: int, theta: float = 500000.0, out=None):
    """qkv = x W_qkv with RoPE applied to the first rope_cols columns (q and k heads)."""
    M, K = x.shape
    N = W_qkv.shape[1]
    _need(x, BF16, "x")
    _need(W_qkv, BF16, "W_qkv", (K, N))
    _need(positions, torch.int32, "positions", (M,))
    if out is None:
        out = _empty((M, N), BF16, x)
    _call("coda_gemm_qkv_rope", _ptr(x), _ptr(W_qkv), _ptr(positions), _ptr(out), M, N, K, int(head_dim),
          int(rope_cols), float(theta), _stream())
    return out


def gemm_swiglu_bwd(d_out, W_down, gateup, out=None):
    """[d_gate | d_up] from d_act = d_out W_down^T and the saved gate/up."""
    M, N = d_out.shape
    F = W_down.shape[0]
    _need(d_out, BF16, "d_out")
    _need(W_down, BF16, "W_down", (F, N))
    _need(gateup, BF16, "gateup", (M, 2 * F))
    if out is None:
        out = _empty((M, 2 * F), BF16, d_out)
    _call("coda_gemm_swiglu_bwd", _ptr(d_out), _ptr(W_down), _ptr(gateup), _ptr(out), M, F, N, _stream())
    return out


def swiglu_mlp_backward(d_h2, y, W_gu, W_down, act, gateup):
    """Backward of h2 = (silu(y W_g) * (y W_u)) W_down + res from the saved
    gate/up and act: returns dict(d_gateup, d_y, dW_gu, dW_down, d_res)."""
    d_gu = gemm_swiglu_bwd(d_h2, W_down, gateup)
    d_y, dW_gu = gemm_res_partialrms_bwd(d_gu, y, W_gu)
    _, dW_down = gemm_res_partialrms_bwd(d_h2, act, W_down, dx=False)
    return {"d_gateup": d_gu, "d_y": d_y, "dW_gu": dW_gu, "dW_down": dW_down, "d_res": d_h2}


def lmhead_ce_workspace_size(M: int, V: int) -> int:
    return int(load_library().coda_lmhead_ce_workspace_size(M, V))


def lmhead_ce(H, W, labels, r=None, ws=None):
    """Fused LM-head cross-entropy; returns (loss[M], lse[M], mean[1]) fp32."""
    M, K = H.shape
    V = W.shape[1]
    _need(H, BF16, "H")
    _need(W, BF16, "W", (K, V))
    _need(labels, torch.int64, "labels", (M,))
    if r is not None:
        _need(r, F32, "r", (M,))
    loss = _empty((M,), F32, H)
    lse = _empty((M,), F32, H)
    mean = _empty((1,), F32, H)
    nb = lmhead_ce_workspace_size(M, V)
    if ws is None:
        ws = _empty((max(nb, 16),), torch.uint8, H)
    _call("coda_lmhead_ce", _ptr(H), _ptr(W), _ptr(labels), _ptr(r), _ptr(loss), _ptr(lse), _ptr(mean),
          _ptr(ws), ws.numel(), M, V, K, _stream())
    return loss, lse, mean


def lmhead_ce_bwd(H, W, labels, lse, d_loss=None, r=None, ws=None):
    """Backward of the fused cross-entropy from the saved lse; returns (dH, dW) fp32.
    d_loss None weights every token by 1/M (the mean)."""
    M, K = H.shape
    V = W.shape[1]
    _need(H, BF16, "H")
    _need(W, BF16, "W", (K, V))
    _need(labels, torch.int64, "labels", (M,))
    _need(lse, F32, "lse", (M,))
    if d_loss is not None:
        _need(d_loss, F32, "d_loss", (M,))
    if r is not None:
        _need(r, F32, "r", (M,))
    dH = _empty((M, K), F32, H)
    dW = _empty((K, V), F32, H)
    nb = int(load_library().coda_lmhead_ce_bwd_workspace_size(M, V))
    if ws is None:
        ws = _empty((max(nb, 16),), torch.uint8, H)
    _call("coda_lmhead_ce_bwd", _ptr(H), _ptr(W), _ptr(labels), _ptr(lse), _ptr(d_loss), _ptr(r), _ptr(dH), _ptr(dW),
          _ptr(ws), ws.numel(), M, V, K, _stream())
    return dH, dW


def loss_stats(loss, stats_out=None):
    """(sum of loss, count) as a [2] fp32 device tensor, for an all-reduce over ranks."""
    _need(loss, F32, "loss")
    stats_out = _empty((2,), F32, loss) if stats_out is None else stats_out
    _call("coda_loss_stats", _ptr(loss), loss.numel(), _ptr(stats_out), _stream())
    return stats_out


def ce_global_finish(stats, M: int, mean=True, d_loss=True):
    """From rank-summed stats: (mean [1] or None, d_loss [M] = 1/count or None)."""
    _need(stats, F32, "stats", (2,))
    mean_out = _empty((1,), F32, stats) if mean else None
    d_out = _empty((M,), F32, stats) if d_loss else None
    _call("coda_ce_global_finish", _ptr(stats), int(M), _ptr(mean_out), _ptr(d_out), _stream())
    return mean_out, d_out


# ---------------------------------------------------------------- backward


def gemm_rowscale_bwd(dOut, hg, W2, r, ws=None):
    """Backward of out = r * (hg W2); returns (d_hg, dW2, pdr)."""
    M, N2 = dOut.shape
    N = hg.shape[1]
    _need(dOut, BF16, "dOut")
    _need(hg, BF16, "hg", (M, N))
    _need(W2, BF16, "W2", (N, N2))
    _need(r, F32, "r", (M,))
    d_hg = _empty((M, N), F32, dOut)
    dW2 = _empty((N, N2), F32, dOut)
    pdr = _empty((partial_cols(N), M), F32, dOut)
    nb = int(load_library().coda_gemm_rowscale_bwd_workspace_size(M, N))
    if ws is None:
        ws = _empty((max(nb, 16),), torch.uint8, dOut)
    _call("coda_gemm_rowscale_bwd", _ptr(dOut), _ptr(hg), _ptr(W2), _ptr(r), _ptr(d_hg), _ptr(dW2), _ptr(pdr),
          _ptr(ws), ws.numel(), M, N, N2, _stream())
    return d_hg, dW2, pdr


def rms_reduce_bwd(pdr, r, d_hg, h, gamma, ws=None):
    """RMSNorm backward row reduction; returns (dh, dgamma)."""
    T, M = pdr.shape
    N = h.shape[1]
    _need(pdr, F32, "pdr")
    _need(r, F32, "r", (M,))
    _need(d_hg, F32, "d_hg", (M, N))
    _need(h, BF16, "h", (M, N))
    _need(gamma, BF16, "gamma", (N,))
    dh = _empty((M, N), BF16, h)
    dgamma = _empty((N,), F32, h)
    nb = int(load_library().coda_rms_reduce_bwd_workspace_size(M, N))
    if ws is None:
        ws = _empty((max(nb, 16),), torch.uint8, h)
    _call("coda_rms_reduce_bwd", _ptr(pdr), _ptr(r), _ptr(d_hg), _ptr(h), _ptr(gamma), _ptr(dh), _ptr(dgamma),
          _ptr(ws), ws.numel(), M, T, N, _stream())
    return dh, dgamma


def gemm_res_partialrms_bwd(dh, x, W1, dx=True, dW1=True):
    """Backward of h = x W1 + res; returns (dx, dW1) (dres is dh)."""
    M, N = dh.shape
    K = x.shape[1]
    _need(dh, BF16, "dh")
    _need(x, BF16, "x", (M, K))
    _need(W1, BF16, "W1", (K, N))
    dx_out = _empty((M, K), BF16, dh) if dx else None
    dW1_out = _empty((K, N), F32, dh) if dW1 else None
    _call("coda_gemm_res_partialrms_bwd", _ptr(dh), _ptr(x), _ptr(W1), _ptr(dx_out), _ptr(dW1_out), M, N, K,
          _stream())
    return dx_out, dW1_out


# ------------------------------------------------------ unfused comparison chain


def unfused_add(a, b, out=None):
    _need(a, BF16, "a")
    _need(b, BF16, "b", tuple(a.shape))
    if out is None:
        out = torch.empty_like(a)
    _call("coda_unfused_add", _ptr(a), _ptr(b), _ptr(out), a.numel(), _stream())
    return out


def unfused_rmsnorm(h, gamma, eps: float, y_out=None, r_out=None):
    M, N = h.shape
    _need(h, BF16, "h")
    _need(gamma, BF16, "gamma", (N,))
    if y_out is None:
        y_out = torch.empty_like(h)
    _call("coda_unfused_rmsnorm", _ptr(h), _ptr(gamma), float(eps), _ptr(y_out), _ptr(r_out), M, N, _stream())
    return y_out


def selftest_bounded_wait(limit_ns: int) -> int:
    """Runs the bounded-wait self test; returns 1 if the wait gave up."""
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")
    _call("coda_selftest_bounded_wait", int(limit_ns), _ptr(flag), _stream())
    torch.cuda.synchronize()
    return int(flag[0].item())


# -------------------------------------------------- call sequences of the path


def rmsnorm_block(x, res, W1, W2, gamma, eps: float, out=None, bufs=None):
    """The whole block in one persistent launch (coda_rmsnorm_block).
    Returns dict(out, h, hg, partial, r)."""
    M, K = x.shape
    N = W1.shape[1]
    N2 = W2.shape[1]
    _need(x, BF16, "x")
    if res is not None:
        _need(res, BF16, "res", (M, N))
    _need(W1, BF16, "W1", (K, N))
    _need(W2, BF16, "W2", (N, N2))
    _need(gamma, BF16, "gamma", (N,))
    b = bufs or {}
    h = b.get("h") if b.get("h") is not None else _empty((M, N), BF16, x)
    hg = b.get("hg") if b.get("hg") is not None else _empty((M, N), BF16, x)
    partial = b.get("partial") if b.get("partial") is not None else _empty((partial_cols(N), M), F32, x)
    r = b.get("r") if b.get("r") is not None else _empty((M,), F32, x)
    if out is None:
        out = _empty((M, N2), BF16, x)
    ws = b.get("ws")
    if ws is None:
        ws = _empty((max(int(load_library().coda_rmsnorm_block_workspace_size(M)), 16),), torch.uint8, x)
    _call("coda_rmsnorm_block", _ptr(x), _ptr(res), _ptr(W1), _ptr(W2), _ptr(gamma), float(eps), _ptr(h), _ptr(hg),
          _ptr(partial), _ptr(r), _ptr(out), _ptr(ws), ws.numel(), M, K, N, N2, _stream())
    return {"out": out, "h": h, "hg": hg, "partial": partial, "r": r}


def gemm_rmsnorm_gemm(x, res, W1, W2, gamma, eps: float, out=None, bufs=None, fold_reduce=True, launches=None):
    """The fused block: first GEMM + residual + partial RMS, the light
    reduction, and the row-scaled second GEMM.  launches=1: one persistent
    launch (coda_rmsnorm_block); 2 (the default, or fold_reduce): the reduction
    inside the second GEMM's epilogue; 3 (fold_reduce=False): the reduction as
    its own kernel.  Returns dict(out, h, hg, partial, r)."""
    if launches is None:
        launches = 2 if fold_reduce else 3
    if launches == 1:
        return rmsnorm_block(x, res, W1, W2, gamma, eps, out=out, bufs=bufs)
    fold_reduce = launches == 2
    N = W1.shape[1]
    b = bufs or {}
    h, hg, partial = gemm_res_partialrms(x, W1, res, gamma, h_out=b.get("h"), hg_out=b.get("hg"),
                                         partial_out=b.get("partial"))
    if fold_reduce:
        out, r = gemm_rowscale_partial(hg, W2, partial, N, eps, out=out, r_out=b.get("r"))
    else:
        r = rms_reduce(partial, N, eps, r_out=b.get("r"))
        out = gemm_rowscale(hg, W2, r, out=out)
    return {"out": out, "h": h, "hg": hg, "partial": partial, "r": r}


# ---------------------------------------------------------------- FP8 (e4m3)

U8 = torch.uint8


def fp8_quantize(src, transpose: bool = False, dst=None, amax=None, scale=None):
    """Per-tensor e4m3 quantisation of a bf16 [rows, cols] tensor (its own
    scale = amax / 448).  Returns (codes uint8 [rows, cols] or, transposed,
    [cols, rows]; amax [1] fp32; scale [1] fp32)."""
    rows, cols = src.shape
    _need(src, BF16, "src")
    if dst is None:
        dst = _empty((cols, rows) if transpose else (rows, cols), U8, src)
    amax = _empty((1,), F32, src) if amax is None else amax
    scale = _empty((1,), F32, src) if scale is None else scale
    _call("coda_fp8_quantize", _ptr(src), rows, cols, 1 if transpose else 0, _ptr(dst), _ptr(amax), _ptr(scale),
          _stream())
    return dst, amax, scale


def fp8_scale_from_amax(amax, scale_out=None):
    """scale = amax / 448 (1 for 0), on the device."""
    _need(amax, F32, "amax", (1,))
    scale_out = _empty((1,), F32, amax) if scale_out is None else scale_out
    _call("coda_fp8_scale_from_amax", _ptr(amax), _ptr(scale_out), _stream())
    return scale_out


def gemm_res_partialrms_fp8(x8, sx, Wt8, sw, res, gamma, s_hg, *, h=True, h_out=None, hg8_out=None,
                            amax_out=None, partial_out=None):
    """First GEMM of the FP8 block.  Returns (h bf16 or None, hg8 e4m3 codes,
    amax [1] = max |gamma * h|, partial [T, M])."""
    M, K = x8.shape
    N = Wt8.shape[0]
    _need(x8, U8, "x8")
    _need(Wt8, U8, "Wt8", (N, K))
    for t, nm in ((sx, "sx"), (sw, "sw"), (s_hg, "s_hg")):
        _need(t, F32, nm, (1,))
    if res is not None:
        _need(res, BF16, "res", (M, N))
    _need(gamma, BF16, "gamma", (N,))
    if h and h_out is None:
        h_out = _empty((M, N), BF16, x8)
    hg8_out = _empty((M, N), U8, x8) if hg8_out is None else hg8_out
    amax_out = _empty((1,), F32, x8) if amax_out is None else amax_out
    partial_out = _empty((partial_cols(N), M), F32, x8) if partial_out is None else partial_out
    _call("coda_gemm_res_partialrms_fp8", _ptr(x8), _ptr(sx), _ptr(Wt8), _ptr(sw), _ptr(res), _ptr(gamma),
          _ptr(s_hg), _ptr(h_out if h else None), _ptr(hg8_out), _ptr(amax_out), _ptr(partial_out), M, N, K,
          _stream())
    return (h_out if h else None), hg8_out, amax_out, partial_out


def gemm_rowscale_partial_fp8(A8, sa, Wt8, sw, partial, N_norm: int, eps: float, out=None, r_out=None):
    """Second GEMM of the FP8 block: out = r * sa * sw * (A8 Wt8^T), r from
    the partials.  Returns (out bf16, r)."""
    M, K = A8.shape
    N = Wt8.shape[0]
    _need(A8, U8, "A8")
    _need(Wt8, U8, "Wt8", (N, K))
    _need(sa, F32, "sa", (1,))
    _need(sw, F32, "sw", (1,))
    _need(partial, F32, "partial", (partial.shape[0], M))
    out = _empty((M, N), BF16, A8) if out is None else out
    r_out = _empty((M,), F32, A8) if r_out is None else r_out
    _call("coda_gemm_rowscale_partial_fp8", _ptr(A8), _ptr(sa), _ptr(Wt8), _ptr(sw), _ptr(partial),
          partial.shape[0], N_norm, float(eps), _ptr(r_out), _ptr(out), M, N, K, _stream())
    return out, r_out


def gemm_rmsnorm_gemm_fp8(x8, sx, W1t8, sw1, res, gamma, s_hg, W2t8, sw2, eps: float, out=None, bufs=None):
    """The FP8 block in two launches (plus the zeroing of amax): returns
    dict(out, h, hg8, amax, partial, r).  s_hg is the scale hg8 is quantised
    with (delayed scaling: fp8_scale_from_amax of an earlier call's amax)."""
    N = W1t8.shape[0]
    b = bufs or {}
    h, hg8, amax, partial = gemm_res_partialrms_fp8(x8, sx, W1t8, sw1, res, gamma, s_hg, h_out=b.get("h"),
                                                    hg8_out=b.get("hg8"), amax_out=b.get("amax"),
                                                    partial_out=b.get("partial"))
    out, r = gemm_rowscale_partial_fp8(hg8, s_hg, W2t8, sw2, partial, N, eps, out=out, r_out=b.get("r"))
    return {"out": out, "h": h, "hg8": hg8, "amax": amax, "partial": partial, "r": r}


def gemm_fp8(A8, sa, Wt8, sw, out=None):
    """out = bf16(sa * sw * (A8 Wt8^T)) with e4m3 A8 [M, K] and Wt8 [N, K]."""
    M, K = A8.shape
    N = Wt8.shape[0]
    _need(A8, U8, "A8")
    _need(Wt8, U8, "Wt8", (N, K))
    _need(sa, F32, "sa", (1,))
    _need(sw, F32, "sw", (1,))
    out = _empty((M, N), BF16, A8) if out is None else out
    _call("coda_gemm_fp8", _ptr(A8), _ptr(sa), _ptr(Wt8), _ptr(sw), _ptr(out), M, N, K, _stream())
    return out


def unfused_rmsnorm_fp8(h, gamma, eps: float, s_y, y8_out=None, amax_out=None, r_out=None):
    """y8 = e4m3(gamma * h * r / s_y), amax = max |y|; returns (y8, amax, r)."""
    M, N = h.shape
    _need(h, BF16, "h")
    _need(gamma, BF16, "gamma", (N,))
    _need(s_y, F32, "s_y", (1,))
    y8_out = _empty((M, N), U8, h) if y8_out is None else y8_out
    amax_out = _empty((1,), F32, h) if amax_out is None else amax_out
    r_out = _empty((M,), F32, h) if r_out is None else r_out
    _call("coda_unfused_rmsnorm_fp8", _ptr(h), _ptr(gamma), float(eps), _ptr(s_y), _ptr(y8_out), _ptr(amax_out),
          _ptr(r_out), M, N, _stream())
    return y8_out, amax_out, r_out


def unfused_block_fp8(x8, sx, W1t8, sw1, res, gamma, s_y, W2t8, sw2, eps: float, out=None, bufs=None):
    """The unfused FP8 chain: FP8 GEMM -> residual add -> RMSNorm with an e4m3
    output -> FP8 GEMM, every intermediate in HBM.  Returns dict(out, t, h,
    y8, amax, r)."""
    b = bufs or {}
    t = gemm_fp8(x8, sx, W1t8, sw1, out=b.get("t"))
    h = unfused_add(t, res, out=b.get("h"))
    y8, amax, r = unfused_rmsnorm_fp8(h, gamma, eps, s_y, y8_out=b.get("y8"), amax_out=b.get("amax"),
                                      r_out=b.get("r"))
    out = gemm_fp8(y8, s_y, W2t8, sw2, out=out)
    return {"out": out, "t": t, "h": h, "y8": y8, "amax": amax, "r": r}


# ----------------------------------------------- block-scaled e4m3 (MXFP8)


MX_A, MX_B = 0, 1  # scale layouts: the GEMM's left operand, its right operand (stored [N, K])


def mx_sf_bytes(rows: int, cols: int, operand: int = MX_A) -> int:
    """Bytes of the scale buffer of a [rows, cols] MXFP8 operand in the
    layout of `operand` (MX_A or MX_B)."""
    n = load_library().coda_mx_sf_bytes(int(rows), int(cols), int(operand))
    if n < 0:
        raise ValueError(f"no MXFP8 layout for [{rows}, {cols}], operand {operand} (cols must be a multiple of 128)")
    return n


def mx_quantize(src, operand: int = MX_A, q_out=None, sf_out=None):
    """MXFP8 codes of a bf16 [rows, cols] tensor, blocked along its rows, with
    its scales in the layout of `operand`.  Returns (codes uint8 [rows, cols],
    scales uint8)."""
    rows, cols = src.shape
    _need(src, BF16, "src")
    q_out = _empty((rows, cols), U8, src) if q_out is None else q_out
    sf_out = _empty((mx_sf_bytes(rows, cols, operand),), U8, src) if sf_out is None else sf_out
    _call("coda_mx_quantize", _ptr(src), rows, cols, int(operand), _ptr(q_out), _ptr(sf_out), _stream())
    return q_out, sf_out


def gemm_res_partialrms_mx(x8, sx, Wt8, sw, res, gamma, *, h=True, h_out=None, hq_out=None, hsf_out=None,
                           partial_out=None):
    """First GEMM of the MXFP8 block.  Returns (h bf16 or None, hg codes,
    hg's scales in the A layout, partial [T, M])."""
    M, K = x8.shape
    N = Wt8.shape[0]
    _need(x8, U8, "x8")
    _need(Wt8, U8, "Wt8", (N, K))
    _need(sx, F32, "sx", (1,))
    _need(sw, F32, "sw", (1,))
    if res is not None:
        _need(res, BF16, "res", (M, N))
    _need(gamma, BF16, "gamma", (N,))
    if h and h_out is None:
        h_out = _empty((M, N), BF16, x8)
    hq_out = _empty((M, N), U8, x8) if hq_out is None else hq_out
    hsf_out = _empty((mx_sf_bytes(M, N, MX_A),), U8, x8) if hsf_out is None else hsf_out
    partial_out = _empty((partial_cols(N), M), F32, x8) if partial_out is None else partial_out
    _call("coda_gemm_res_partialrms_mx", _ptr(x8), _ptr(sx), _ptr(Wt8), _ptr(sw), _ptr(res), _ptr(gamma),
          _ptr(h_out if h else None), _ptr(hq_out), _ptr(hsf_out), _ptr(partial_out), M, N, K, _stream())
    return (h_out if h else None), hq_out, hsf_out, partial_out


def gemm_rowscale_partial_mx(Aq, Asf, Wq, Wsf, partial=None, N_norm: int = 0, eps: float = 0.0, out=None,
                             r_out=None):
    """Second GEMM of the MXFP8 block: out = r * (A Wt^T) with block-scaled
    operands (Asf in the A layout, Wsf in the B layout), r from the partials
    (partial None: a plain MXFP8 GEMM, r = 1).  Returns (out bf16, r or None)."""
    M, K = Aq.shape
    N = Wq.shape[0]
    _need(Aq, U8, "Aq")
    _need(Wq, U8, "Wq", (N, K))
    _need(Asf, U8, "Asf", (mx_sf_bytes(M, K, MX_A),))
    _need(Wsf, U8, "Wsf", (mx_sf_bytes(N, K, MX_B),))
    out = _empty((M, N), BF16, Aq) if out is None else out
    T = 0
    if partial is not None:
        _need(partial, F32, "partial", (partial.shape[0], M))
        T = partial.shape[0]
        r_out = _empty((M,), F32, Aq) if r_out is None else r_out
    else:
        r_out = None
    _call("coda_gemm_rowscale_partial_mx", _ptr(Aq), _ptr(Asf), _ptr(Wq), _ptr(Wsf), _ptr(partial), T, N_norm,
          float(eps), _ptr(r_out), _ptr(out), M, N, K, _stream())
    return out, r_out


def gemm_rmsnorm_gemm_mx(x8, sx, W1t8, sw1, res, gamma, W2q, W2sf, eps: float, out=None, bufs=None):
    """The MXFP8 block in two launches: returns dict(out, h, hq, hsf,
    partial, r).  hg's scales are formed in the first GEMM's epilogue."""
    N = W1t8.shape[0]
    b = bufs or {}
    h, hq, hsf, partial = gemm_res_partialrms_mx(x8, sx, W1t8, sw1, res, gamma, h_out=b.get("h"),
                                                 hq_out=b.get("hq"), hsf_out=b.get("hsf"),
                                                 partial_out=b.get("partial"))
    out, r = gemm_rowscale_partial_mx(hq, hsf, W2q, W2sf, partial, N, eps, out=out, r_out=b.get("r"))
    return {"out": out, "h": h, "hq": hq, "hsf": hsf, "partial": partial, "r": r}


def unfused_block_mx(x8, sx, W1t8, sw1, res, gamma, W2q, W2sf, eps: float, out=None, bufs=None):
    """The unfused MXFP8 chain: FP8 GEMM -> residual add -> RMSNorm (bf16 y) ->
    MXFP8 quantisation of y -> block-scaled GEMM, every intermediate in HBM.
    Returns dict(out, t, h, y, yq, ysf, r)."""
    b = bufs or {}
    M = x8.shape[0]
    t = gemm_fp8(x8, sx, W1t8, sw1, out=b.get("t"))
    h = unfused_add(t, res, out=b.get("h"))
    r = b.get("r")
    if r is None:
        r = _empty((M,), F32, x8)
    y = unfused_rmsnorm(h, gamma, eps, y_out=b.get("y"), r_out=r)
    yq, ysf = mx_quantize(y, MX_A, q_out=b.get("yq"), sf_out=b.get("ysf"))
    out, _ = gemm_rowscale_partial_mx(yq, ysf, W2q, W2sf, out=out)
    return {"out": out, "t": t, "h": h, "y": y, "yq": yq, "ysf": ysf, "r": r}


def _need_host(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def rmsnorm_block_host(x_host, res_host, W1, W2, gamma, eps: float, out_host=None, chunk_rows: int = 512,
                       ws=None):
    """The block with host-resident x, res and out (pin them for overlap);
    weights on the device.  Rows stream through in chunks whose copies in
    and out overlap the compute.  Returns out_host (complete once the
    current stream is synchronised)."""
    M, K = x_host.shape
    N = W1.shape[1]
    N2 = W2.shape[1]
    _need_host(x_host, BF16, "x_host")
    if res_host is not None:
        _need_host(res_host, BF16, "res_host", (M, N))
    _need(W1, BF16, "W1", (K, N))
    _need(W2, BF16, "W2", (N, N2))
    _need(gamma, BF16, "gamma", (N,))
    if out_host is None:
        out_host = torch.empty((M, N2), dtype=BF16, pin_memory=True)
    _need_host(out_host, BF16, "out_host", (M, N2))
    nb = int(load_library().coda_rmsnorm_block_host_workspace_size(K, N, N2, chunk_rows))
    if ws is None:
        ws = _empty((max(nb, 16),), torch.uint8, W1)
    _call("coda_rmsnorm_block_host", x_host.data_ptr(), None if res_host is None else res_host.data_ptr(), _ptr(W1),
          _ptr(W2), _ptr(gamma), float(eps), out_host.data_ptr(), _ptr(ws), ws.numel(), M, K, N, N2, chunk_rows,
          _stream())
    return out_host


def unfused_block(x, res, W1, W2, gamma, eps: float, out=None, bufs=None):
    """The unfused comparison chain: GEMM -> add -> RMSNorm -> GEMM, each
    intermediate written to and read back from HBM."""
    b = bufs or {}
    t = gemm_rowscale(x, W1, None, out=b.get("t"))
    h = unfused_add(t, res, out=b.get("h"))
    y = unfused_rmsnorm(h, gamma, eps, y_out=b.get("y"))
    out = gemm_rowscale(y, W2, None, out=out)
    return {"out": out, "h": h, "y": y}


def swiglu_down(hg, r, h, W_gu, W_down, save=False):
    """SwiGLU + down projection + residual + partials for the next norm."""
    act, gu = gemm_swiglu(hg, W_gu, r, save=save)
    h2, _, partial2 = gemm_res_partialrms(act, W_down, h, None, hg=False)
    return {"act": act, "gateup": gu, "h2": h2, "partial2": partial2}


def block_backward(dOut, x, W1, W2, gamma, fwd):
    """Backward of the fused block from its saved state (h, hg, r)."""
    d_hg, dW2, pdr = gemm_rowscale_bwd(dOut, fwd["hg"], W2, fwd["r"])
    dh, dgamma = rms_reduce_bwd(pdr, fwd["r"], d_hg, fwd["h"], gamma)
    dx, dW1 = gemm_res_partialrms_bwd(dh, x, W1)
    return {"dW2": dW2, "dgamma": dgamma, "dh": dh, "dres": dh, "dx": dx, "dW1": dW1, "d_hg": d_hg, "pdr": pdr}
