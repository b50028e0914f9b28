"""Python binding of ``libfp8w8a8.so`` (the C ABI in ``include/fp8w8a8.h``).

Argument marshalling only: every step of the W8A8 path runs in the library's
CUDA kernels. PyTorch provides device memory and the current stream. Importing
this package fails loudly if the compiled library is missing; there is no CPU
fallback.

Functions mirror the C entry points:

* :func:`repack_qat` - QAT q4_0 grid -> per-channel E4M3 weight + scales.
* :func:`convert_fnuz` - E4M3FNUZ-stored weight -> E4M3 weight + scales.
* :func:`quant_act` - per-token E4M3 activation quantization.
* :func:`rowwise_linear` - ``y = (x8 . w8^T) * s_tok * s_ch`` in bf16;
  :func:`rowwise_linear_ws` with a workspace (:func:`linear_workspace`).
* :func:`linear` - bf16 activations in, bf16 out (quantizer + GEMM).
* :func:`linear_siblings` - several linears of the same x, quantized once.
* :func:`cast_e4m3` - the element-wise encoder.
* :func:`moe_route`, :func:`moe_gather`, :func:`grouped_linear`,
  :func:`moe_geglu_quant`, :func:`moe_combine` - the mixture-of-experts layer.
* :func:`bf16_linear` - the bf16 GEMM (the router), :func:`moe_topk` - the
  router's top-k choice and weights.
* :func:`w4a16_dequant`, :func:`w4a16_linear` - the W4A16 build (int4 QAT
  weights, bf16 activations).
* :func:`int8_repack_qat`, :func:`int8_quant_act`, :func:`int8_rowwise_linear`
  (:func:`int8_rowwise_linear_ws` with a workspace),
  :func:`int8_linear` - the int8 W8A8 build.
* :func:`device_status` - read and clear the device status word.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8w8a8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python fp8_w8a8_linear_b200/build.py` "
        "(the FP8 W8A8 path has no fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "fp8_version": ([], ctypes.c_int),
    "fp8_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "fp8_device_supported": ([ctypes.c_int], ctypes.c_int),
    "fp8_get_device_status": ([ctypes.POINTER(ctypes.c_uint)], ctypes.c_int),
    "fp8_test_set_fault": ([_I64, ctypes.c_int32], ctypes.c_int),
    "fp8_repack_qat": ([_P, _P, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "fp8_convert_fnuz": ([_P, _P, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "fp8_quant_act": ([_P, _I64, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "fp8_rowwise_linear": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], ctypes.c_int),
    "fp8_linear_workspace_bytes": ([], ctypes.c_size_t),
    "fp8_rowwise_linear_ws": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "fp8_linear_bf16": ([_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
    "fp8_cast_e4m3": ([_P, _I64, _P, _P], ctypes.c_int),
    "fp8_linear_bf16_siblings": ([_P, _I64, _I64, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P],
                                 ctypes.c_int),
    "fp8_linear_bf16_noalloc": ([_P, _P, _P, _I64, _I64, _I64, _P, _P], ctypes.c_int),
    "fp8_moe_route": ([_P, _I64, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P], ctypes.c_int),
    "fp8_moe_gather": ([_P, _P, _P, _I64, _I64, ctypes.c_int32, _P, _P, _P], ctypes.c_int),
    "fp8_grouped_linear": ([_P, _P, _P, ctypes.c_int32, _I64, _P, _P, _I64, _I64, _P, _P],
                           ctypes.c_int),
    "fp8_moe_geglu_quant": ([_P, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
    "fp8_moe_interleave_gate_up": ([_P, _P, ctypes.c_int32, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "fp8_grouped_linear_geglu": ([_P, _P, _P, ctypes.c_int32, _I64, _P, _P, _I64, _I64, _P, _P],
                                 ctypes.c_int),
    "fp8_moe_combine": ([_P, _P, _I64, ctypes.c_int32, _I64, _P, _P, _P], ctypes.c_int),
    "bf16_linear": ([_P, _P, _I64, _I64, _I64, _P, _P], ctypes.c_int),
    "fp8_moe_topk": ([_P, _I64, ctypes.c_int32, ctypes.c_int32, _P, _P, _P], ctypes.c_int),
    "w4a16_dequant": ([_P, _P, _I64, _I64, _P, _P], ctypes.c_int),
    "w4a16_workspace_bytes": ([_I64, _I64, _I64], ctypes.c_size_t),
    "w4a16_linear": ([_P, _P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "int8_repack_qat": ([_P, _P, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "int8_quant_act": ([_P, _I64, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "int8_rowwise_linear": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], ctypes.c_int),
    "int8_rowwise_linear_ws": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "int8_linear_bf16": ([_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _ret

raw = _lib  # the C entry points themselves (plain pointers and sizes)

FP8_OK = 0
DEV_NONFINITE = 0x1
DEV_NAN_CODE = 0x2
DEV_INEXACT = 0x4
DEV_TIMEOUT = 0x8
DEV_BAD_INDEX = 0x10


class Fp8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_lib.fp8_status_string(status).decode()} ({status})")
        self.status = status


def _check(status: int, where: str):
    if status != FP8_OK:
        raise Fp8Error(status, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, dtype, name: str, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def version() -> int:
    return _lib.fp8_version()


def device_supported(device: int = 0) -> bool:
    return bool(_lib.fp8_device_supported(device))


def device_status() -> int:
    """Synchronize the current device, return its status bits and clear them."""
    v = ctypes.c_uint(0)
    _check(_lib.fp8_get_device_status(ctypes.byref(v)), "fp8_get_device_status")
    return v.value


def test_set_fault(wait_cycles: int = 0, drop_step: int = -1):
    """Test hook: in-kernel wait limit (0 = default) and the decode GEMM's
    dropped pipeline step (-1 = none); see fp8_test_set_fault."""
    _check(_lib.fp8_test_set_fault(wait_cycles, drop_step), "fp8_test_set_fault")


def repack_qat(q4: torch.Tensor, d: torch.Tensor, w8: torch.Tensor | None = None,
               s_ch: torch.Tensor | None = None):
    """q4 uint8 [N, K/2] (packed int4) and d float32 [N, K/32] -> (w8 uint8 [N, K], s_ch float32 [N])."""
    N, K2 = q4.shape
    K = 2 * K2
    w8 = torch.empty((N, K), dtype=torch.uint8, device=q4.device) if w8 is None else w8
    s_ch = torch.empty((N,), dtype=torch.float32, device=q4.device) if s_ch is None else s_ch
    _check(_lib.fp8_repack_qat(_dev(q4, torch.uint8, "q4"), _dev(d, torch.float32, "d", (N, K // 32)),
                               N, K, _dev(w8, torch.uint8, "w8", (N, K)),
                               _dev(s_ch, torch.float32, "s_ch", (N,)), _stream()), "fp8_repack_qat")
    return w8, s_ch


def convert_fnuz(w8_fnuz: torch.Tensor, s_fnuz: torch.Tensor, w8: torch.Tensor | None = None,
                 s_ch: torch.Tensor | None = None):
    """E4M3FNUZ codes [N, K] + scales [N] -> E4M3 codes + scales (in place if outputs alias)."""
    N, K = w8_fnuz.shape
    w8 = torch.empty_like(w8_fnuz) if w8 is None else w8
    s_ch = torch.empty_like(s_fnuz) if s_ch is None else s_ch
    _check(_lib.fp8_convert_fnuz(_dev(w8_fnuz, torch.uint8, "w8_fnuz"),
                                 _dev(s_fnuz, torch.float32, "s_fnuz", (N,)), N, K,
                                 _dev(w8, torch.uint8, "w8", (N, K)),
                                 _dev(s_ch, torch.float32, "s_ch", (N,)), _stream()),
           "fp8_convert_fnuz")
    return w8, s_ch


def quant_act(x: torch.Tensor, x8: torch.Tensor | None = None, s_tok: torch.Tensor | None = None):
    """x bf16 [M, K] -> (x8 uint8 [M, K], s_tok float32 [M])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with unit inner stride")
    M, K = x.shape
    x8 = torch.empty((M, K), dtype=torch.uint8, device=x.device) if x8 is None else x8
    s_tok = torch.empty((M,), dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    _check(_lib.fp8_quant_act(x.data_ptr(), M, K, x.stride(0), _dev(x8, torch.uint8, "x8", (M, K)),
                              _dev(s_tok, torch.float32, "s_tok", (M,)), _stream()), "fp8_quant_act")
    return x8, s_tok


def rowwise_linear(x8: torch.Tensor, s_tok: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor,
                   y: torch.Tensor | None = None):
    """y bf16 [M, N] = (x8 . w8^T) * s_tok[:, None] * s_ch[None, :]."""
    M, K = x8.shape
    N = w8.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x8.device) if y is None else y
    _check(_lib.fp8_rowwise_linear(_dev(x8, torch.uint8, "x8"), _dev(s_tok, torch.float32, "s_tok", (M,)),
                                   _dev(w8, torch.uint8, "w8", (N, K)),
                                   _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                   _dev(y, torch.bfloat16, "y", (M, N)), _stream()),
           "fp8_rowwise_linear")
    return y


def linear_workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for rowwise_linear_ws on the current device
    (uint8, fp8_linear_workspace_bytes() bytes; at least 16)."""
    n = int(_lib.fp8_linear_workspace_bytes())
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def rowwise_linear_ws(x8: torch.Tensor, s_tok: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor,
                      ws: torch.Tensor, y: torch.Tensor | None = None):
    """rowwise_linear with a workspace (from linear_workspace) that lets a
    partial last wave of tiles be split by k-blocks over all SM pairs."""
    M, K = x8.shape
    N = w8.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x8.device) if y is None else y
    _check(_lib.fp8_rowwise_linear_ws(_dev(x8, torch.uint8, "x8"), _dev(s_tok, torch.float32, "s_tok", (M,)),
                                      _dev(w8, torch.uint8, "w8", (N, K)),
                                      _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                      _dev(y, torch.bfloat16, "y", (M, N)), _dev(ws, torch.uint8, "ws"),
                                      ws.numel(), _stream()),
           "fp8_rowwise_linear_ws")
    return y


def linear(x: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor, y: torch.Tensor | None = None,
           x8: torch.Tensor | None = None, s_tok: torch.Tensor | None = None):
    """The W8A8 linear from bf16 activations: quantize per token, then GEMM."""
    M, K = x.shape
    N = w8.shape[0]
    dev = x.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    x8 = torch.empty((M, K), dtype=torch.uint8, device=dev) if x8 is None else x8
    s_tok = torch.empty((M,), dtype=torch.float32, device=dev) if s_tok is None else s_tok
    _check(_lib.fp8_linear_bf16(_dev(x, torch.bfloat16, "x"), _dev(w8, torch.uint8, "w8", (N, K)),
                                _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                _dev(x8, torch.uint8, "x8", (M, K)),
                                _dev(s_tok, torch.float32, "s_tok", (M,)),
                                _dev(y, torch.bfloat16, "y", (M, N)), _stream()), "fp8_linear_bf16")
    return y


def linear_siblings(x: torch.Tensor, weights, ys=None, x8: torch.Tensor | None = None,
                    s_tok: torch.Tensor | None = None):
    """Several W8A8 linears of the same bf16 activations (q/k/v, gate/up):
    x is quantized once. ``weights`` is a list of (w8 [N_i, K], s_ch [N_i])."""
    M, K = x.shape
    dev = x.device
    n = len(weights)
    ys = [torch.empty((M, w.shape[0]), dtype=torch.bfloat16, device=dev) for w, _ in weights] if ys is None else ys
    x8 = torch.empty((M, K), dtype=torch.uint8, device=dev) if x8 is None else x8
    s_tok = torch.empty((M,), dtype=torch.float32, device=dev) if s_tok is None else s_tok
    P = ctypes.c_void_p * n
    w_arr = P(*[_dev(w, torch.uint8, "w8", (w.shape[0], K)) for w, _ in weights])
    s_arr = P(*[_dev(sc, torch.float32, "s_ch", (w.shape[0],)) for w, sc in weights])
    n_arr = (ctypes.c_int64 * n)(*[w.shape[0] for w, _ in weights])
    y_arr = P(*[_dev(yy, torch.bfloat16, "y", (M, w.shape[0])) for yy, (w, _) in zip(ys, weights)])
    _check(_lib.fp8_linear_bf16_siblings(_dev(x, torch.bfloat16, "x"), M, K, n, ctypes.cast(w_arr, _P),
                                         ctypes.cast(s_arr, _P), ctypes.cast(n_arr, _P),
                                         _dev(x8, torch.uint8, "x8", (M, K)),
                                         _dev(s_tok, torch.float32, "s_tok", (M,)),
                                         ctypes.cast(y_arr, _P), _stream()), "fp8_linear_bf16_siblings")
    return ys


# ------------------------------------------------------------------ MoE
def moe_route(topk_ids: torch.Tensor, num_experts: int):
    """topk_ids int32 [T, k] -> (perm [T*k], inv [T*k], offsets [E+1]) int32."""
    T, k = topk_ids.shape
    dev = topk_ids.device
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    _check(_lib.fp8_moe_route(_dev(topk_ids, torch.int32, "topk_ids"), T, k, num_experts,
                              perm.data_ptr(), inv.data_ptr(), offsets.data_ptr(), _stream()),
           "fp8_moe_route")
    return perm, inv, offsets


def moe_gather(x8: torch.Tensor, s_tok: torch.Tensor, perm: torch.Tensor, top_k: int,
               x8_rows: torch.Tensor | None = None, s_rows: torch.Tensor | None = None):
    rows = perm.numel()
    K = x8.shape[1]
    x8_rows = torch.empty((rows, K), dtype=torch.uint8, device=x8.device) if x8_rows is None else x8_rows
    s_rows = torch.empty((rows,), dtype=torch.float32, device=x8.device) if s_rows is None else s_rows
    _check(_lib.fp8_moe_gather(_dev(x8, torch.uint8, "x8"), _dev(s_tok, torch.float32, "s_tok"),
                               _dev(perm, torch.int32, "perm"), rows, K, top_k,
                               _dev(x8_rows, torch.uint8, "x8_rows", (rows, K)),
                               _dev(s_rows, torch.float32, "s_rows", (rows,)), _stream()),
           "fp8_moe_gather")
    return x8_rows, s_rows


def grouped_linear(x8_rows: torch.Tensor, s_rows: torch.Tensor, offsets: torch.Tensor,
                   w8: torch.Tensor, s_ch: torch.Tensor, y: torch.Tensor | None = None):
    """Per-expert GEMM: w8 [E, N, K] (or stacked [E*N, K]), s_ch [E, N] or [E*N]."""
    M, K = x8_rows.shape
    E = offsets.numel() - 1
    N = w8.numel() // (E * K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x8_rows.device) if y is None else y
    _check(_lib.fp8_grouped_linear(_dev(x8_rows, torch.uint8, "x8_rows"),
                                   _dev(s_rows, torch.float32, "s_rows", (M,)),
                                   _dev(offsets, torch.int32, "offsets"), E, M,
                                   _dev(w8, torch.uint8, "w8"), _dev(s_ch, torch.float32, "s_ch"),
                                   N, K, _dev(y, torch.bfloat16, "y", (M, N)), _stream()),
           "fp8_grouped_linear")
    return y


def moe_interleave_gate_up(w8: torch.Tensor, s_ch: torch.Tensor, num_experts: int, inter: int,
                           w8_il: torch.Tensor | None = None, s_il: torch.Tensor | None = None):
    """Gate/up weights [E, 2*inter, K] -> the interleaved layout of
    grouped_linear_geglu: [E, 256*ceil(inter/128), K] and its scales."""
    E = num_experts
    K = w8.numel() // (E * 2 * inter)
    rows = 256 * ((inter + 127) // 128)
    dev = w8.device
    w8_il = torch.empty((E * rows, K), dtype=torch.uint8, device=dev) if w8_il is None else w8_il
    s_il = torch.empty((E * rows,), dtype=torch.float32, device=dev) if s_il is None else s_il
    _check(_lib.fp8_moe_interleave_gate_up(_dev(w8, torch.uint8, "w8"), _dev(s_ch, torch.float32, "s_ch"),
                                           E, inter, K, _dev(w8_il, torch.uint8, "w8_il"),
                                           _dev(s_il, torch.float32, "s_il"), _stream()),
           "fp8_moe_interleave_gate_up")
    return w8_il, s_il


def grouped_linear_geglu(x8_rows: torch.Tensor, s_rows: torch.Tensor, offsets: torch.Tensor,
                         w8_il: torch.Tensor, s_il: torch.Tensor, inter: int,
                         h: torch.Tensor | None = None):
    """Expert gate/up GEMM with the GeGLU unit in its epilogue: h [M, inter] bf16."""
    M, K = x8_rows.shape
    E = offsets.numel() - 1
    h = torch.empty((M, inter), dtype=torch.bfloat16, device=x8_rows.device) if h is None else h
    _check(_lib.fp8_grouped_linear_geglu(_dev(x8_rows, torch.uint8, "x8_rows"),
                                         _dev(s_rows, torch.float32, "s_rows", (M,)),
                                         _dev(offsets, torch.int32, "offsets"), E, M,
                                         _dev(w8_il, torch.uint8, "w8_il"),
                                         _dev(s_il, torch.float32, "s_il"), inter, K,
                                         _dev(h, torch.bfloat16, "h", (M, inter)), _stream()),
           "fp8_grouped_linear_geglu")
    return h


def moe_geglu_quant(gate_up: torch.Tensor, inter: int, h8=None, s_h=None, h_out=None):
    M = gate_up.shape[0]
    dev = gate_up.device
    h8 = torch.empty((M, inter), dtype=torch.uint8, device=dev) if h8 is None else h8
    s_h = torch.empty((M,), dtype=torch.float32, device=dev) if s_h is None else s_h
    _check(_lib.fp8_moe_geglu_quant(_dev(gate_up, torch.bfloat16, "gate_up", (M, 2 * inter)), M, inter,
                                    _dev(h8, torch.uint8, "h8", (M, inter)),
                                    _dev(s_h, torch.float32, "s_h", (M,)),
                                    None if h_out is None else _dev(h_out, torch.bfloat16, "h_out", (M, inter)),
                                    _stream()), "fp8_moe_geglu_quant")
    return h8, s_h


def moe_combine(rows: torch.Tensor, inv: torch.Tensor, tokens: int, top_k: int,
                weights: torch.Tensor | None = None, out: torch.Tensor | None = None):
    H = rows.shape[1]
    out = torch.empty((tokens, H), dtype=torch.bfloat16, device=rows.device) if out is None else out
    _check(_lib.fp8_moe_combine(_dev(rows, torch.bfloat16, "rows"), _dev(inv, torch.int32, "inv"), tokens,
                                top_k, H, None if weights is None else _dev(weights, torch.float32, "weights"),
                                _dev(out, torch.bfloat16, "out", (tokens, H)), _stream()), "fp8_moe_combine")
    return out


def bf16_linear(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None):
    """y bf16 [M, N] = x [M, K] . w [N, K]^T with bf16 operands (fp32 accumulation)."""
    M, K = x.shape
    N = w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(_lib.bf16_linear(_dev(x, torch.bfloat16, "x"), _dev(w, torch.bfloat16, "w", (N, K)), M, N, K,
                            _dev(y, torch.bfloat16, "y", (M, N)), _stream()), "bf16_linear")
    return y


def moe_topk(logits: torch.Tensor, top_k: int, ids: torch.Tensor | None = None,
             weights: torch.Tensor | None = None):
    """Router logits bf16 [T, E] -> (ids int32 [T, k], weights fp32 [T, k])."""
    T, E = logits.shape
    dev = logits.device
    ids = torch.empty((T, top_k), dtype=torch.int32, device=dev) if ids is None else ids
    weights = torch.empty((T, top_k), dtype=torch.float32, device=dev) if weights is None else weights
    _check(_lib.fp8_moe_topk(_dev(logits, torch.bfloat16, "logits"), T, E, top_k,
                             _dev(ids, torch.int32, "ids", (T, top_k)),
                             _dev(weights, torch.float32, "weights", (T, top_k)), _stream()),
           "fp8_moe_topk")
    return ids, weights


# ------------------------------------------------------------------ W4A16
def w4a16_dequant(q4: torch.Tensor, d: torch.Tensor, w: torch.Tensor | None = None):
    """q4 uint8 [N, K/2] + d float32 [N, K/32] -> w bf16 [N, K] = bf16(fp32(d * q))."""
    N, K2 = q4.shape
    K = 2 * K2
    w = torch.empty((N, K), dtype=torch.bfloat16, device=q4.device) if w is None else w
    _check(_lib.w4a16_dequant(_dev(q4, torch.uint8, "q4"), _dev(d, torch.float32, "d", (N, K // 32)), N, K,
                              _dev(w, torch.bfloat16, "w", (N, K)), _stream()), "w4a16_dequant")
    return w


def w4a16_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.w4a16_workspace_bytes(M, N, K))


def w4a16_linear(x: torch.Tensor, q4: torch.Tensor, d: torch.Tensor, y: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None):
    """y bf16 [M, N] = x bf16 [M, K] . w^T with w the int4 QAT weights unpacked
    to bf16 (in the kernel for M <= 64, else into the workspace ws)."""
    M, K = x.shape
    N = q4.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    need = w4a16_workspace_bytes(M, N, K)
    if need and ws is None:
        ws = torch.empty((N, K), dtype=torch.bfloat16, device=x.device)
    ws_ptr = None if ws is None else ws.data_ptr()
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.w4a16_linear(_dev(x, torch.bfloat16, "x"), _dev(q4, torch.uint8, "q4", (N, K // 2)),
                             _dev(d, torch.float32, "d", (N, K // 32)), M, N, K,
                             _dev(y, torch.bfloat16, "y", (M, N)), ws_ptr, ws_bytes, _stream()),
           "w4a16_linear")
    return y


# ------------------------------------------------------------------ int8 W8A8
def int8_repack_qat(q4: torch.Tensor, d: torch.Tensor, w8: torch.Tensor | None = None,
                    s_ch: torch.Tensor | None = None):
    """q4 uint8 [N, K/2] and d float32 [N, K/32] -> (w8 int8 [N, K], s_ch float32 [N])."""
    N, K2 = q4.shape
    K = 2 * K2
    w8 = torch.empty((N, K), dtype=torch.int8, device=q4.device) if w8 is None else w8
    s_ch = torch.empty((N,), dtype=torch.float32, device=q4.device) if s_ch is None else s_ch
    _check(_lib.int8_repack_qat(_dev(q4, torch.uint8, "q4"), _dev(d, torch.float32, "d", (N, K // 32)),
                                N, K, _dev(w8, torch.int8, "w8", (N, K)),
                                _dev(s_ch, torch.float32, "s_ch", (N,)), _stream()), "int8_repack_qat")
    return w8, s_ch


def int8_quant_act(x: torch.Tensor, x8: torch.Tensor | None = None, s_tok: torch.Tensor | None = None):
    """x bf16 [M, K] -> (x8 int8 [M, K], s_tok float32 [M])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1 or not x.is_cuda:
        raise ValueError("x must be a CUDA bf16 [M, K] tensor with unit inner stride")
    M, K = x.shape
    x8 = torch.empty((M, K), dtype=torch.int8, device=x.device) if x8 is None else x8
    s_tok = torch.empty((M,), dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _check(_lib.int8_quant_act(x.data_ptr(), M, K, x.stride(0), _dev(x8, torch.int8, "x8", (M, K)),
                               _dev(s_tok, torch.float32, "s_tok", (M,)), _stream()), "int8_quant_act")
    return x8, s_tok


def int8_rowwise_linear(x8: torch.Tensor, s_tok: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor,
                        y: torch.Tensor | None = None):
    """y bf16 [M, N] = (x8 . w8^T) * s_tok[:, None] * s_ch[None, :] with int8 operands."""
    M, K = x8.shape
    N = w8.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x8.device) if y is None else y
    _check(_lib.int8_rowwise_linear(_dev(x8, torch.int8, "x8"), _dev(s_tok, torch.float32, "s_tok", (M,)),
                                    _dev(w8, torch.int8, "w8", (N, K)),
                                    _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                    _dev(y, torch.bfloat16, "y", (M, N)), _stream()),
           "int8_rowwise_linear")
    return y


def int8_rowwise_linear_ws(x8: torch.Tensor, s_tok: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor,
                           ws: torch.Tensor, y: torch.Tensor | None = None):
    """int8_rowwise_linear with a workspace (from linear_workspace) for the
    k-block split; bit-identical to int8_rowwise_linear."""
    M, K = x8.shape
    N = w8.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x8.device) if y is None else y
    _check(_lib.int8_rowwise_linear_ws(_dev(x8, torch.int8, "x8"), _dev(s_tok, torch.float32, "s_tok", (M,)),
                                       _dev(w8, torch.int8, "w8", (N, K)),
                                       _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                       _dev(y, torch.bfloat16, "y", (M, N)), _dev(ws, torch.uint8, "ws"),
                                       ws.numel(), _stream()),
           "int8_rowwise_linear_ws")
    return y


def int8_linear(x: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor, y: torch.Tensor | None = None,
                x8: torch.Tensor | None = None, s_tok: torch.Tensor | None = None):
    """The int8 W8A8 linear from bf16 activations: int8 quant per token, then GEMM."""
    M, K = x.shape
    N = w8.shape[0]
    dev = x.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    x8 = torch.empty((M, K), dtype=torch.int8, device=dev) if x8 is None else x8
    s_tok = torch.empty((M,), dtype=torch.float32, device=dev) if s_tok is None else s_tok
    _check(_lib.int8_linear_bf16(_dev(x, torch.bfloat16, "x"), _dev(w8, torch.int8, "w8", (N, K)),
                                 _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                 _dev(x8, torch.int8, "x8", (M, K)),
                                 _dev(s_tok, torch.float32, "s_tok", (M,)),
                                 _dev(y, torch.bfloat16, "y", (M, N)), _stream()), "int8_linear_bf16")
    return y


NOALLOC_SCRATCH_BYTES = 4 << 20


def linear_noalloc(x: torch.Tensor, w8: torch.Tensor, s_ch: torch.Tensor,
                   y: torch.Tensor | None = None):
    """Same result as :func:`linear`, with the quantized activations kept in
    the library's fixed device scratch array instead of caller buffers (for
    callers that cannot allocate device memory). Problems needing more than
    ``NOALLOC_SCRATCH_BYTES`` of scratch raise ``Fp8Error``. Calls that can
    overlap on the GPU share that scratch and must be serialized."""
    M, K = x.shape
    N = w8.shape[0]
    if y is None:
        raise ValueError("pass a preallocated y: this entry point is for callers that do not allocate")
    _check(_lib.fp8_linear_bf16_noalloc(_dev(x, torch.bfloat16, "x"), _dev(w8, torch.uint8, "w8", (N, K)),
                                        _dev(s_ch, torch.float32, "s_ch", (N,)), M, N, K,
                                        _dev(y, torch.bfloat16, "y", (M, N)), _stream()),
           "fp8_linear_bf16_noalloc")
    return y


def cast_e4m3(x: torch.Tensor, out: torch.Tensor | None = None):
    """Element-wise fp32 -> E4M3 codes with the library's encoder."""
    n = x.numel()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    _check(_lib.fp8_cast_e4m3(_dev(x, torch.float32, "x"), n, _dev(out, torch.uint8, "out"), _stream()),
           "fp8_cast_e4m3")
    return out


__all__ = [
    "Fp8Error", "raw", "version", "device_supported", "device_status", "repack_qat",
    "convert_fnuz", "quant_act", "rowwise_linear", "rowwise_linear_ws", "linear_workspace", "linear",
    "linear_noalloc", "cast_e4m3",
    "linear_siblings", "test_set_fault",
    "moe_route", "moe_gather", "grouped_linear", "moe_geglu_quant", "moe_combine",
    "moe_interleave_gate_up", "grouped_linear_geglu",
    "int8_repack_qat", "int8_quant_act", "int8_rowwise_linear", "int8_rowwise_linear_ws", "int8_linear",
    "bf16_linear", "moe_topk", "w4a16_dequant", "w4a16_workspace_bytes", "w4a16_linear",
    "DEV_NONFINITE", "DEV_NAN_CODE", "DEV_INEXACT", "DEV_TIMEOUT", "LIB_PATH",
]
