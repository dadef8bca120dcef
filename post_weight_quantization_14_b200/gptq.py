"""Thin ctypes binding of the C ABI in include/gptq_b200.h.

Argument marshalling only: every computation runs in the CUDA kernels of
``libgptq_b200.so``.  PyTorch supplies device memory and the current stream.
The functions keep the C names; ``quantize_layer`` chains the three stages for
one linear layer (the call a user makes).
"""

from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgptq_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gptq_b200.h")

GPTQ_OK = 0
GPTQ_ERR_INVALID_ARG = 1
GPTQ_ERR_UNSUPPORTED = 2
GPTQ_ERR_NOT_PD = 3
GPTQ_ERR_NONFINITE = 4
GPTQ_ERR_CUDA = 5
GPTQ_ERR_TIMEOUT = 6
GPTQ_ERR_WORKSPACE = 7

GPTQ_BF16 = 0
GPTQ_F32 = 1


class GptqConfig(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int), ("sym", ctypes.c_int),
                ("block_size", ctypes.c_int), ("damp_rel", ctypes.c_float), ("desc_act", ctypes.c_int)]


class GPTQError(RuntimeError):
    def __init__(self, status: int, msg: str, index: int | None = None):
        super().__init__(f"{msg} (status {status})")
        self.status = status
        self.index = index


_lib = None
_vp, _i64, _sz, _int, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float

_SIGS = {
    "gptq_default_config": (None, [ctypes.POINTER(GptqConfig)]),
    "gptq_status_string": (ctypes.c_char_p, [_int]),
    "gptq_last_error": (ctypes.c_char_p, []),
    "gptq_version": (_int, []),
    "gptq_hessian_workspace_bytes": (_sz, [_i64, _i64, _int]),
    "gptq_hessian_accumulate": (_int, [_vp, _int, _i64, _i64, _vp, _int, _vp, _sz, _vp]),
    "gptq_prepare_hinv_workspace_bytes": (_sz, [_i64]),
    "gptq_prepare_hinv": (_int, [_vp, _i64, _f32, _vp, _vp, _sz, ctypes.POINTER(_i64),
                                 ctypes.POINTER(_f32), _vp]),
    "gptq_prepare_hinv_async": (_int, [_vp, _i64, _f32, _vp, _vp, _sz, _vp, _vp]),
    "gptq_prepare_hinv_permuted_async": (_int, [_vp, _vp, _i64, _f32, _vp, _vp, _sz, _vp, _vp]),
    "gptq_quantize_workspace_bytes": (_sz, [_i64, _i64, ctypes.POINTER(GptqConfig)]),
    "gptq_quantize_layer": (_int, [_vp, _vp, _i64, _i64, ctypes.POINTER(GptqConfig), _vp, _vp, _vp, _vp,
                                   _vp, _sz, _vp]),
    "gptq_pack_int": (_int, [_vp, _i64, _i64, _int, _int, _vp, _vp]),
    "gptq_dequant": (_int, [_vp, _vp, _vp, _i64, _i64, ctypes.POINTER(GptqConfig), _vp, _vp]),
    "gptq_sync_status": (_int, [_vp]),
    "gptq_timing_enable": (None, [_int]),
    "gptq_timing_report": (_sz, [ctypes.c_char_p, _sz]),
    "gptq_timing_timeline": (_sz, [ctypes.c_char_p, _sz]),
    "gptq_chol_schedule": (_i64, [_i64, ctypes.c_void_p, _i64]),
    "gptq_selftest_bounded_wait": (_int, [ctypes.c_uint64, _vp]),
    "gptq_hessian_accumulate_fixed_scratch": (_int, [_vp, _int, _i64, _i64, _vp, _int, _vp]),
    "gptq_act_sum_accumulate": (_int, [_vp, _int, _i64, _i64, _vp, _int, _vp]),
    "gptq_act_order": (_int, [_vp, _i64, _int, _vp, _vp, _vp]),
    "gptq_prepare_hinv_permuted": (_int, [_vp, _vp, _i64, _f32, _vp, _vp, _sz, ctypes.POINTER(_i64),
                                          ctypes.POINTER(_f32), _vp]),
    "gptq_quantize_layer_act_order": (_int, [_vp, _vp, _vp, _i64, _i64, ctypes.POINTER(GptqConfig), _vp, _vp, _vp,
                                             _vp, _vp, _vp, _sz, _vp]),
    "gptq_dequant_g_idx": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, ctypes.POINTER(GptqConfig), _vp, _vp]),
    "gptq_dequant_gemm": (_int, [_vp, _i64, _vp, _vp, _vp, _i64, _i64, ctypes.POINTER(GptqConfig), _vp, _vp]),
    "gptq_layer_loss_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "gptq_layer_loss": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "gptq_2d_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "gptq_2d_round": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _sz, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libgptq_b200.so (fails loudly when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m post_weight_quantization_14_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/gptq_b200.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z0-9_]+)\s*\(", text)))


ACT_ASCENDING = 1    # desc_act = 1: ascending sum of |x|, least influential columns first
ACT_DESCENDING = 2   # desc_act = 2: descending


def make_config(bits=4, group_size=128, sym=False, block_size=128, damp_rel=0.01, desc_act=0) -> GptqConfig:
    """desc_act: 0 natural order, 1 ascending and 2 descending activation order (True means 1)."""
    c = GptqConfig()
    lib().gptq_default_config(ctypes.byref(c))
    c.bits, c.group_size, c.sym, c.block_size = int(bits), int(group_size), int(bool(sym)), int(block_size)
    c.damp_rel, c.desc_act = float(damp_rel), int(desc_act)
    return c


def _check(status: int, index: int | None = None) -> None:
    if status != GPTQ_OK:
        msg = lib().gptq_last_error().decode()
        raise GPTQError(status, msg or lib().gptq_status_string(status).decode(), index)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------- stage wrappers

_WORD = (torch.int32, torch.uint32)   # packed 32-bit words: either signedness


def _need(t: torch.Tensor, dtype, shape: tuple, name: str, flat_ok: bool = False) -> None:
    """Shape and dtype check before any pointer reaches the library (the C side sees only
    addresses and sizes, so a mismatch here would be an out-of-range access on the device).
    dtype may be a tuple of accepted dtypes; flat_ok also accepts a 1-D tensor of the
    same number of elements."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    dtypes = dtype if isinstance(dtype, tuple) else (dtype,)
    numel = 1
    for x in shape:
        numel *= int(x)
    shape_ok = tuple(t.shape) == tuple(shape) or (flat_ok and t.dim() == 1 and t.numel() == numel)
    if t.dtype not in dtypes or not shape_ok:
        raise ValueError(f"{name} must be {dtypes[0]} {list(shape)} (got {t.dtype} {list(t.shape)})")


def _quant_outputs(cfg: GptqConfig, d_out: int, d_in: int, qweight, scales, qzeros, err_sq) -> None:
    """Shapes and dtypes of the column loop's output arrays (layouts of include/gptq_b200.h)."""
    ng = n_groups(d_in, cfg.group_size)
    _need(qweight, _WORD, ((d_in * cfg.bits + 31) // 32, d_out), "qweight")
    _need(scales, torch.float16, (ng, d_out), "scales")
    if cfg.sym:
        if qzeros is not None:
            raise ValueError("qzeros must be None for symmetric quantization")
    else:
        if qzeros is None:
            raise ValueError("qzeros is required for asymmetric quantization")
        _need(qzeros, _WORD, (ng, (d_out * cfg.bits + 31) // 32), "qzeros")
    if err_sq is not None:
        _need(err_sq, torch.float32, (d_out,), "err_sq")


def gptq_hessian_accumulate(X: torch.Tensor, H: torch.Tensor, accumulate: bool = False,
                            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H (+)= 2 X^T X.  X: [n, d_in] bfloat16 or float32 on the device; H: [d_in, d_in] float32."""
    if X.dim() != 2:
        raise ValueError("X must be a [n, d_in] matrix")
    n, d_in = X.shape
    if X.dtype == torch.bfloat16:
        xt = GPTQ_BF16
    elif X.dtype == torch.float32:
        xt = GPTQ_F32
    else:
        raise ValueError("X must be bfloat16 or float32")
    if H.dtype != torch.float32 or tuple(H.shape) != (d_in, d_in):
        raise ValueError("H must be float32 [d_in, d_in]")
    need = lib().gptq_hessian_workspace_bytes(n, d_in, xt)
    ws = workspace if workspace is not None else _workspace(need, X.device)
    _check(lib().gptq_hessian_accumulate(_ptr(X), xt, n, d_in, _ptr(H), int(bool(accumulate)),
                                         _ptr(ws), ws.numel(), _stream(stream)))
    return H


def gptq_prepare_hinv(H: torch.Tensor, U: torch.Tensor, damp_rel: float = 0.01,
                      workspace: torch.Tensor | None = None, stream=None) -> float:
    """U = upper Cholesky factor of (H + lambda I)^-1; returns lambda.  Synchronises the stream."""
    if H.dim() != 2:
        raise ValueError("H must be a square float32 matrix")
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(U, torch.float32, (d, d), "U")
    need = lib().gptq_prepare_hinv_workspace_bytes(d)
    ws = workspace if workspace is not None else _workspace(need, H.device)
    bad = _i64(-1)
    lam = _f32(0.0)
    st = lib().gptq_prepare_hinv(_ptr(H), d, float(damp_rel), _ptr(U), _ptr(ws), ws.numel(),
                                 ctypes.byref(bad), ctypes.byref(lam), _stream(stream))
    _check(st, bad.value)
    return float(lam.value)


def gptq_prepare_hinv_async(H: torch.Tensor, U: torch.Tensor, damp_rel: float = 0.01,
                            workspace: torch.Tensor | None = None, lam: torch.Tensor | None = None,
                            perm: torch.Tensor | None = None, stream=None) -> None:
    """U as gptq_prepare_hinv (of H[perm][:, perm] when perm is given) with no host
    synchronisation; lam (float32 [1] on the device, optional) receives lambda.  Errors
    surface at the next gptq_sync_status()."""
    if H.dim() != 2:
        raise ValueError("H must be a square float32 matrix")
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(U, torch.float32, (d, d), "U")
    if lam is not None:
        _need(lam, torch.float32, (1,), "lam")
    need = lib().gptq_prepare_hinv_workspace_bytes(d)
    ws = workspace if workspace is not None else _workspace(need, H.device)
    if perm is None:
        _check(lib().gptq_prepare_hinv_async(_ptr(H), d, float(damp_rel), _ptr(U), _ptr(ws), ws.numel(), _ptr(lam),
                                             _stream(stream)))
    else:
        _need(perm, torch.int32, (d,), "perm")
        _check(lib().gptq_prepare_hinv_permuted_async(_ptr(H), _ptr(perm), d, float(damp_rel), _ptr(U), _ptr(ws),
                                                      ws.numel(), _ptr(lam), _stream(stream)))


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, cfg: GptqConfig, qweight: torch.Tensor,
                        scales: torch.Tensor, qzeros: torch.Tensor | None, err_sq: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None) -> None:
    """Column loop; W is consumed as scratch.  scales is a float16 tensor [n_groups, d_out]."""
    if W.dim() != 2:
        raise ValueError("W must be a float32 [d_out, d_in] matrix")
    d_out, d_in = W.shape
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(U, torch.float32, (d_in, d_in), "U")
    _quant_outputs(cfg, d_out, d_in, qweight, scales, qzeros, err_sq)
    need = lib().gptq_quantize_workspace_bytes(d_out, d_in, ctypes.byref(cfg))
    ws = workspace if workspace is not None else _workspace(need, W.device)
    _check(lib().gptq_quantize_layer(_ptr(W), _ptr(U), d_out, d_in, ctypes.byref(cfg), _ptr(qweight),
                                     _ptr(scales), _ptr(qzeros), _ptr(err_sq), _ptr(ws), ws.numel(),
                                     _stream(stream)))


def gptq_act_sum_accumulate(X: torch.Tensor, act: torch.Tensor, accumulate: bool = False, stream=None) -> torch.Tensor:
    """act[c] (+)= sum_t |X[t, c]| (fp64).  X: [n, d_in] bfloat16 or float32; act: float64 [d_in]."""
    n, d_in = X.shape
    xt = GPTQ_BF16 if X.dtype == torch.bfloat16 else GPTQ_F32 if X.dtype == torch.float32 else None
    if xt is None:
        raise ValueError("X must be bfloat16 or float32")
    if act.dtype != torch.float64 or tuple(act.shape) != (d_in,):
        raise ValueError("act must be float64 [d_in]")
    _check(lib().gptq_act_sum_accumulate(_ptr(X), xt, n, d_in, _ptr(act), int(bool(accumulate)), _stream(stream)))
    return act


def gptq_act_order(act: torch.Tensor, desc_act: int, perm: torch.Tensor, rank: torch.Tensor, stream=None) -> None:
    """perm[k] = column quantized at position k, rank = its inverse (int32 [d_in] each)."""
    d = act.numel()
    _need(act, torch.float64, (d,), "act")
    _need(perm, torch.int32, (d,), "perm")
    _need(rank, torch.int32, (d,), "rank")
    _check(lib().gptq_act_order(_ptr(act), act.numel(), int(desc_act), _ptr(perm), _ptr(rank), _stream(stream)))


def gptq_prepare_hinv_permuted(H: torch.Tensor, perm: torch.Tensor, U: torch.Tensor, damp_rel: float = 0.01,
                               workspace: torch.Tensor | None = None, stream=None) -> float:
    """U of the permuted Hessian H[perm][:, perm]; returns lambda.  Synchronises the stream."""
    d = H.shape[0]
    _need(H, torch.float32, (d, d), "H")
    _need(perm, torch.int32, (d,), "perm")
    _need(U, torch.float32, (d, d), "U")
    need = lib().gptq_prepare_hinv_workspace_bytes(d)
    ws = workspace if workspace is not None else _workspace(need, H.device)
    bad = _i64(-1)
    lam = _f32(0.0)
    st = lib().gptq_prepare_hinv_permuted(_ptr(H), _ptr(perm), d, float(damp_rel), _ptr(U), _ptr(ws), ws.numel(),
                                          ctypes.byref(bad), ctypes.byref(lam), _stream(stream))
    _check(st, bad.value)
    return float(lam.value)


def gptq_quantize_layer_act_order(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor, cfg: GptqConfig,
                                  qweight: torch.Tensor, scales: torch.Tensor, qzeros: torch.Tensor | None,
                                  g_idx: torch.Tensor, err_sq: torch.Tensor | None = None,
                                  workspace: torch.Tensor | None = None, stream=None) -> None:
    """Column loop in the order perm (cfg.desc_act 1 or 2); W is read only; codes in original order."""
    if W.dim() != 2:
        raise ValueError("W must be a float32 [d_out, d_in] matrix")
    d_out, d_in = W.shape
    _need(W, torch.float32, (d_out, d_in), "W")
    _need(U, torch.float32, (d_in, d_in), "U")
    _need(perm, torch.int32, (d_in,), "perm")
    _need(g_idx, torch.int32, (d_in,), "g_idx")
    _quant_outputs(cfg, d_out, d_in, qweight, scales, qzeros, err_sq)
    need = lib().gptq_quantize_workspace_bytes(d_out, d_in, ctypes.byref(cfg))
    ws = workspace if workspace is not None else _workspace(need, W.device)
    _check(lib().gptq_quantize_layer_act_order(_ptr(W), _ptr(U), _ptr(perm), d_out, d_in, ctypes.byref(cfg),
                                               _ptr(qweight), _ptr(scales), _ptr(qzeros), _ptr(g_idx), _ptr(err_sq),
                                               _ptr(ws), ws.numel(), _stream(stream)))


def gptq_dequant_g_idx(qweight, scales, qzeros, g_idx, d_out: int, d_in: int, cfg: GptqConfig, W_hat: torch.Tensor,
                       stream=None) -> torch.Tensor:
    _quant_outputs(cfg, d_out, d_in, qweight, scales, qzeros, None)
    _need(g_idx, torch.int32, (d_in,), "g_idx")
    _need(W_hat, torch.float32, (d_out, d_in), "W_hat")
    _check(lib().gptq_dequant_g_idx(_ptr(qweight), _ptr(scales), _ptr(qzeros), _ptr(g_idx), d_out, d_in,
                                    ctypes.byref(cfg), _ptr(W_hat), _stream(stream)))
    return W_hat


def gptq_dequant_gemm(X: torch.Tensor, qweight, scales, qzeros, d_out: int, d_in: int, cfg: GptqConfig,
                      Y: torch.Tensor, stream=None) -> torch.Tensor:
    """Y = X W_hat^T from the packed arrays.  X: bfloat16 [M, d_in]; Y: float32 [M, d_out]."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != d_in:
        raise ValueError("X must be bfloat16 [M, d_in]")
    if Y.dtype != torch.float32 or tuple(Y.shape) != (X.shape[0], d_out):
        raise ValueError("Y must be float32 [M, d_out]")
    _quant_outputs(cfg, d_out, d_in, qweight, scales, qzeros, None)
    _check(lib().gptq_dequant_gemm(_ptr(X), X.shape[0], _ptr(qweight), _ptr(scales), _ptr(qzeros), d_out, d_in,
                                   ctypes.byref(cfg), _ptr(Y), _stream(stream)))
    return Y


def gptq_layer_loss(W: torch.Tensor, W_hat: torch.Tensor, X: torch.Tensor, row_loss: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """E = ||(W - W_hat) X^T||_F^2 on the device: a float64 [1] tensor (not synchronised).
    W, W_hat: float32 [d_out, d_in]; X: bfloat16 or float32 [n, d_in]; row_loss, when given,
    float64 [d_out] receives each row's part."""
    if W.dim() != 2 or X.dim() != 2 or W.shape[1] != X.shape[1]:
        raise ValueError("W must be [d_out, d_in] and X [n, d_in]")
    d_out, d_in = W.shape
    if W.dtype != torch.float32 or W_hat.dtype != torch.float32 or tuple(W_hat.shape) != (d_out, d_in):
        raise ValueError("W and W_hat must be float32 [d_out, d_in]")
    xt = GPTQ_BF16 if X.dtype == torch.bfloat16 else GPTQ_F32 if X.dtype == torch.float32 else None
    if xt is None:
        raise ValueError("X must be bfloat16 or float32")
    if row_loss is not None and (row_loss.dtype != torch.float64 or tuple(row_loss.shape) != (d_out,)):
        raise ValueError("row_loss must be float64 [d_out]")
    n = X.shape[0]
    need = lib().gptq_layer_loss_workspace_bytes(d_out, d_in, n)
    ws = workspace if workspace is not None else _workspace(need, W.device)
    loss = torch.empty((1,), dtype=torch.float64, device=W.device)
    _check(lib().gptq_layer_loss(_ptr(W), _ptr(W_hat), _ptr(X), xt, d_out, d_in, n, _ptr(row_loss), _ptr(loss),
                                 _ptr(ws), ws.numel(), _stream(stream)))
    return loss


def gptq_2d_round(X: torch.Tensor, U_left: torch.Tensor, U_right: torch.Tensor, Z: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """GPTQ-2D two-sided rounding.  X: float64 [m, n] or [batch, m, n]; U_left float64 [m, m],
    U_right float64 [n, n] (upper Cholesky factors of the inverse Grams); returns Z int32 of
    X's shape."""
    if X.dim() not in (2, 3):
        raise ValueError("X must be [m, n] or [batch, m, n]")
    batch = 1 if X.dim() == 2 else X.shape[0]
    m, n = X.shape[-2], X.shape[-1]
    _need(X, torch.float64, tuple(X.shape), "X")
    _need(U_left, torch.float64, (m, m), "U_left")
    _need(U_right, torch.float64, (n, n), "U_right")
    if Z is None:
        Z = torch.empty(X.shape, dtype=torch.int32, device=X.device)
    _need(Z, torch.int32, tuple(X.shape), "Z")
    need = lib().gptq_2d_workspace_bytes(m, n, batch)
    ws = workspace if workspace is not None else _workspace(need, X.device)
    _check(lib().gptq_2d_round(_ptr(X), m, n, batch, _ptr(U_left), _ptr(U_right), _ptr(Z), _ptr(ws), ws.numel(),
                               _stream(stream)))
    return Z


def gptq_pack_int(codes: torch.Tensor, bits: int, layout: int, packed: torch.Tensor, stream=None) -> torch.Tensor:
    """codes uint8 [rows, cols] -> packed int32 ([rows, nwords] for layout 0, [nwords, rows] for 1)."""
    if codes.dim() != 2:
        raise ValueError("codes must be a uint8 [rows, cols] matrix")
    rows, cols = codes.shape
    nw = (cols * int(bits) + 31) // 32
    _need(codes, torch.uint8, (rows, cols), "codes")
    _need(packed, _WORD, (rows, nw) if layout == 0 else (nw, rows), "packed", flat_ok=True)
    _check(lib().gptq_pack_int(_ptr(codes), rows, cols, int(bits), int(layout), _ptr(packed), _stream(stream)))
    return packed


def gptq_dequant(qweight, scales, qzeros, d_out: int, d_in: int, cfg: GptqConfig, W_hat: torch.Tensor,
                 stream=None) -> torch.Tensor:
    _quant_outputs(cfg, d_out, d_in, qweight, scales, qzeros, None)
    _need(W_hat, torch.float32, (d_out, d_in), "W_hat")
    _check(lib().gptq_dequant(_ptr(qweight), _ptr(scales), _ptr(qzeros), d_out, d_in, ctypes.byref(cfg),
                              _ptr(W_hat), _stream(stream)))
    return W_hat


def gptq_sync_status(stream=None) -> None:
    _check(lib().gptq_sync_status(_stream(stream)))


def gptq_timing_enable(on: bool = True) -> None:
    lib().gptq_timing_enable(int(bool(on)))


def gptq_timing_report() -> dict:
    """{kernel: (launches, total_ms)} since the last report (synchronises the device)."""
    import json
    n = lib().gptq_timing_report(None, 0)
    buf = ctypes.create_string_buffer(n + 16)
    lib().gptq_timing_report(buf, len(buf))
    return {k: (int(v[0]), float(v[1])) for k, v in json.loads(buf.value.decode()).items()}


def gptq_timing_timeline() -> list:
    """[(kernel, stream_index, start_ms, end_ms), ...] of the launches recorded since the last
    collection (synchronises the device)."""
    import json
    n = lib().gptq_timing_timeline(None, 0)
    buf = ctypes.create_string_buffer(n + 16)
    lib().gptq_timing_timeline(buf, len(buf))
    return [tuple(x) for x in json.loads(buf.value.decode())]


def gptq_chol_schedule(T: int) -> list:
    """The factorization kernel's product order for T tiles per side: [(type, a, b, c), ...]
    (host-side; the encoding is the one include/gptq_b200.h gives)."""
    total = lib().gptq_chol_schedule(int(T), None, 0)
    if total < 0:
        raise GPTQError(int(GPTQ_ERR_INVALID_ARG), f"T out of range ({T})")
    buf = (ctypes.c_int32 * (4 * total))()
    lib().gptq_chol_schedule(int(T), buf, total)
    return [tuple(buf[4 * t:4 * t + 4]) for t in range(total)]


def gptq_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(lib().gptq_selftest_bounded_wait(int(limit_ns), _stream(stream)))


# ---------------------------------------------------------------------------- whole layer

def n_groups(d_in: int, group_size: int) -> int:
    return 1 if group_size == -1 else (d_in + group_size - 1) // group_size


def _resolve_config(buffers, bits, group_size, sym, damp_rel, desc_act) -> GptqConfig:
    """The configuration of a whole-layer call.  Without buffers the arguments give it (None
    means the default: 4 bits, group 128, asymmetric, damp 0.01, natural order).  With
    buffers the buffers' configuration is used, and an argument given explicitly that
    disagrees with it is an error rather than silently ignored."""
    given = dict(bits=bits, group_size=group_size, sym=sym, damp_rel=damp_rel, desc_act=desc_act)
    if buffers is None:
        d = dict(bits=4, group_size=128, sym=False, damp_rel=0.01, desc_act=0)
        d.update({k: v for k, v in given.items() if v is not None})
        return make_config(d["bits"], d["group_size"], d["sym"], 128, d["damp_rel"], d["desc_act"])
    cfg = buffers.cfg
    have = dict(bits=cfg.bits, group_size=cfg.group_size, sym=bool(cfg.sym), damp_rel=cfg.damp_rel,
                desc_act=cfg.desc_act)
    for k, v in given.items():
        if v is None:
            continue
        same = abs(float(v) - have[k]) <= 1e-7 * max(1.0, abs(have[k])) if k == "damp_rel" else \
            (bool(v) == have[k] if k == "sym" else int(v) == have[k])
        if not same:
            raise ValueError(f"{k}={v!r} conflicts with the buffers' configuration ({k}={have[k]!r})")
    return cfg


@dataclass
class QuantizedLayer:
    qweight: torch.Tensor      # int32 [ceil(d_in*bits/32), d_out]
    scales: torch.Tensor       # float16 [n_groups, d_out]
    qzeros: torch.Tensor | None  # int32 [n_groups, ceil(d_out*bits/32)] (None if sym)
    err_sq: torch.Tensor       # float32 [d_out]
    lam: float
    g_idx: torch.Tensor | None = None   # int32 [d_in] with activation ordering
    perm: torch.Tensor | None = None    # int32 [d_in] quantization order


class LayerBuffers:
    """Device buffers for one layer shape, reusable across calls (no allocation per call)."""

    def __init__(self, d_out: int, d_in: int, n: int, x_dtype: torch.dtype, cfg: GptqConfig, device):
        xt = GPTQ_BF16 if x_dtype == torch.bfloat16 else GPTQ_F32
        L = lib()
        self.cfg = cfg
        self.H = torch.empty((d_in, d_in), dtype=torch.float32, device=device)
        self.U = torch.empty((d_in, d_in), dtype=torch.float32, device=device)
        self.lam = torch.zeros((1,), dtype=torch.float32, device=device)
        ws = max(L.gptq_hessian_workspace_bytes(n, d_in, xt), L.gptq_prepare_hinv_workspace_bytes(d_in),
                 L.gptq_quantize_workspace_bytes(d_out, d_in, ctypes.byref(cfg)))
        self.ws = _workspace(ws, device)
        ng = n_groups(d_in, cfg.group_size)
        self.qweight = torch.empty(((d_in * cfg.bits + 31) // 32, d_out), dtype=torch.int32, device=device)
        self.scales = torch.empty((ng, d_out), dtype=torch.float16, device=device)
        self.qzeros = None if cfg.sym else torch.empty((ng, (d_out * cfg.bits + 31) // 32), dtype=torch.int32,
                                                      device=device)
        self.err_sq = torch.empty((d_out,), dtype=torch.float32, device=device)
        if cfg.desc_act:
            self.act = torch.empty((d_in,), dtype=torch.float64, device=device)
            self.perm = torch.empty((d_in,), dtype=torch.int32, device=device)
            self.rank = torch.empty((d_in,), dtype=torch.int32, device=device)
            self.g_idx = torch.empty((d_in,), dtype=torch.int32, device=device)


def quantize_layer(W: torch.Tensor, X: torch.Tensor, bits=None, group_size=None, sym=None, damp_rel=None,
                   desc_act=None, buffers: LayerBuffers | None = None, stream=None) -> QuantizedLayer:
    """GPTQ of one linear layer: H = 2 X^T X, U = chol(Hd^-1) upper, column loop.

    desc_act 0: natural column order, W is overwritten.  desc_act 1 / 2: columns in
    ascending / descending order of sum_t |X[t, c]|; W is left unchanged and the result
    carries g_idx and perm.

    With ``buffers`` the configuration is the buffers' own (an explicit argument that
    disagrees raises ValueError), and the returned tensors ARE the buffers' arrays: they
    stay valid only until the next call with the same buffers, which overwrites them."""
    cfg = _resolve_config(buffers, bits, group_size, sym, damp_rel, desc_act)
    d_out, d_in = W.shape
    b = buffers or LayerBuffers(d_out, d_in, X.shape[0], X.dtype, cfg, W.device)
    # the three stages are enqueued without a host round trip; one synchronisation at the end
    # reports any device-detected error (a non-positive pivot, non-finite values)
    gptq_hessian_accumulate(X, b.H, accumulate=False, workspace=b.ws, stream=stream)
    if not cfg.desc_act:
        gptq_prepare_hinv_async(b.H, b.U, cfg.damp_rel, workspace=b.ws, lam=b.lam, stream=stream)
        gptq_quantize_layer(W, b.U, cfg, b.qweight, b.scales, b.qzeros, b.err_sq, workspace=b.ws, stream=stream)
        gptq_sync_status(stream)
        return QuantizedLayer(b.qweight, b.scales, b.qzeros, b.err_sq, float(b.lam.item()))
    gptq_act_sum_accumulate(X, b.act, accumulate=False, stream=stream)
    gptq_act_order(b.act, cfg.desc_act, b.perm, b.rank, stream=stream)
    gptq_prepare_hinv_async(b.H, b.U, cfg.damp_rel, workspace=b.ws, lam=b.lam, perm=b.perm, stream=stream)
    gptq_quantize_layer_act_order(W, b.U, b.perm, cfg, b.qweight, b.scales, b.qzeros, b.g_idx, b.err_sq,
                                  workspace=b.ws, stream=stream)
    gptq_sync_status(stream)
    return QuantizedLayer(b.qweight, b.scales, b.qzeros, b.err_sq, float(b.lam.item()), b.g_idx, b.perm)


class SharedInputBuffers:
    """Device buffers for several layers that read the same calibration input X (for
    example the q, k and v projections, or gate and up): one H, one U, one workspace
    large enough for the widest layer, and per-layer outputs."""

    def __init__(self, d_outs: list[int], d_in: int, n: int, x_dtype: torch.dtype, cfg: GptqConfig, device):
        xt = GPTQ_BF16 if x_dtype == torch.bfloat16 else GPTQ_F32
        L = lib()
        self.cfg = cfg
        self.d_in = d_in
        self.H = torch.empty((d_in, d_in), dtype=torch.float32, device=device)
        self.U = torch.empty((d_in, d_in), dtype=torch.float32, device=device)
        ws = max([L.gptq_hessian_workspace_bytes(n, d_in, xt), L.gptq_prepare_hinv_workspace_bytes(d_in)] +
                 [L.gptq_quantize_workspace_bytes(d, d_in, ctypes.byref(cfg)) for d in d_outs])
        self.ws = _workspace(ws, device)
        ng = n_groups(d_in, cfg.group_size)
        self.outs = []
        for d in d_outs:
            self.outs.append(dict(
                qweight=torch.empty(((d_in * cfg.bits + 31) // 32, d), dtype=torch.int32, device=device),
                scales=torch.empty((ng, d), dtype=torch.float16, device=device),
                qzeros=None if cfg.sym else torch.empty((ng, (d * cfg.bits + 31) // 32), dtype=torch.int32,
                                                        device=device),
                err_sq=torch.empty((d,), dtype=torch.float32, device=device),
                g_idx=torch.empty((d_in,), dtype=torch.int32, device=device) if cfg.desc_act else None))
        if cfg.desc_act:
            self.act = torch.empty((d_in,), dtype=torch.float64, device=device)
            self.perm = torch.empty((d_in,), dtype=torch.int32, device=device)
            self.rank = torch.empty((d_in,), dtype=torch.int32, device=device)


def quantize_layers_shared_input(Ws: list[torch.Tensor], X: torch.Tensor, bits=None, group_size=None, sym=None,
                                 damp_rel=None, desc_act=None, buffers: SharedInputBuffers | None = None,
                                 stream=None) -> list[QuantizedLayer]:
    """GPTQ of several linear layers that share one input: H = 2 X^T X, the activation order
    (desc_act 1 / 2) and U = chol(Hd^-1) upper are computed once, then one column loop runs
    per weight.  Each result equals quantize_layer of that weight with the same X.  With
    desc_act 0 every W is overwritten; with activation ordering they are left unchanged.

    With ``buffers`` the configuration is the buffers' own (an explicit argument that
    disagrees raises ValueError), and the returned tensors ARE the buffers' arrays
    (buffers.outs, buffers.perm): they stay valid only until the next call with the same
    buffers, which overwrites them."""
    if not Ws:
        return []
    d_in = Ws[0].shape[1]
    if any(W.shape[1] != d_in for W in Ws) or X.shape[1] != d_in:
        raise ValueError("all weights must have d_in columns, X must be [n, d_in]")
    cfg = _resolve_config(buffers, bits, group_size, sym, damp_rel, desc_act)
    b = buffers or SharedInputBuffers([W.shape[0] for W in Ws], d_in, X.shape[0], X.dtype, cfg, Ws[0].device)
    if len(b.outs) != len(Ws) or any(o["err_sq"].shape[0] != W.shape[0] for o, W in zip(b.outs, Ws)):
        raise ValueError("buffers were made for other layer shapes")
    gptq_hessian_accumulate(X, b.H, accumulate=False, workspace=b.ws, stream=stream)
    if cfg.desc_act:
        gptq_act_sum_accumulate(X, b.act, accumulate=False, stream=stream)
        gptq_act_order(b.act, cfg.desc_act, b.perm, b.rank, stream=stream)
        lam = gptq_prepare_hinv_permuted(b.H, b.perm, b.U, cfg.damp_rel, workspace=b.ws, stream=stream)
    else:
        lam = gptq_prepare_hinv(b.H, b.U, cfg.damp_rel, workspace=b.ws, stream=stream)
    results = []
    for W, o in zip(Ws, b.outs):
        if cfg.desc_act:
            gptq_quantize_layer_act_order(W, b.U, b.perm, cfg, o["qweight"], o["scales"], o["qzeros"], o["g_idx"],
                                          o["err_sq"], workspace=b.ws, stream=stream)
            results.append(QuantizedLayer(o["qweight"], o["scales"], o["qzeros"], o["err_sq"], lam, o["g_idx"],
                                          b.perm))
        else:
            gptq_quantize_layer(W, b.U, cfg, o["qweight"], o["scales"], o["qzeros"], o["err_sq"], workspace=b.ws,
                                stream=stream)
            results.append(QuantizedLayer(o["qweight"], o["scales"], o["qzeros"], o["err_sq"], lam))
    return results
