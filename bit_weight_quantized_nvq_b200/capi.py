"""Thin Python binding of the C ABI in ``include/nvq.h`` (ctypes).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libnvq.so``.  PyTorch provides device memory and streams.  If
the library has not been built, importing this module raises ImportError: no
entry point has a CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libnvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m bit_weight_quantized_nvq_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_c_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class Linear(ctypes.Structure):
    """``nvq_linear``: one NVFP4 weight matrix in device memory."""
    _fields_ = [("codes", _vp), ("scales", _vp), ("g", ctypes.c_float),
                ("N", _c_i64), ("K", _c_i64)]


STACK_LINEARS = 7

#: every symbol the C header declares, with (restype, argtypes)
SIGNATURES = {
    "nvq_version": (ctypes.c_int, []),
    "nvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nvq_last_cuda_error": (ctypes.c_char_p, []),
    "nvq_pack_nvfp4": (ctypes.c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _vp]),
    "nvq_quantize_act_q8_0": (ctypes.c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _vp]),
    "nvq_gemv": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _vp,
                                _c_i64, _vp, _vp]),
    "nvq_gemv_requant": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp]),
    "nvq_gemv_grouped": (ctypes.c_int, [ctypes.POINTER(Linear), _c_i64, _vp, _vp, _c_i64,
                                        ctypes.POINTER(_vp), _vp]),
    "nvq_moe_gemv": (ctypes.c_int, [_vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _vp, _c_i64, _c_i64,
                                    _vp, _vp, _vp, _vp]),
    "nvq_gemm_workspace_size": (ctypes.c_size_t, [_c_i64, _c_i64, _c_i64]),
    "nvq_gemm_w4a16_workspace_size": (ctypes.c_size_t, [_c_i64, _c_i64, _c_i64]),
    "nvq_gemm_w4a16": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _c_i64, _vp,
                                      _vp, ctypes.c_size_t, _vp]),
    "nvq_gemm": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _vp,
                                _c_i64, _vp, _vp, ctypes.c_size_t, _vp]),
    "nvq_quantize_act_nvfp4": (ctypes.c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _vp, _vp]),
    "nvq_gemm_nvf4": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _vp, _vp,
                                     _c_i64, _vp, _vp]),
    "nvq_gemm_noalloc": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp, _vp,
                                        _c_i64, _vp, _vp]),
    "nvq_debug_subblock_sums": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _c_i64, _c_i64, _vp,
                                               _vp, _c_i64, _vp, _vp, _vp]),
    "nvq_error_flags": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]),
    "nvq_debug_stalled_wait": (ctypes.c_int, [ctypes.c_uint64, _vp, _vp]),
    "nvq_decoder_stack": (ctypes.c_int, [ctypes.POINTER(Linear), _c_i64, _vp, _c_i64,
                                         ctypes.POINTER(_vp), _vp, ctypes.c_size_t, _vp]),
    "nvq_decoder_stack_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Linear), _c_i64]),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

NVQ_OK = 0
NVQ_ERR_INVALID_ARG = 1
NVQ_ERR_BAD_SHAPE = 2
NVQ_ERR_MISALIGNED = 3
NVQ_ERR_CUDA = 4
NVQ_ERR_UNSUPPORTED_DEVICE = 5
NVQ_ERR_WORKSPACE = 6


class NVQError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, func: str, status: int):
        self.status = status
        msg = _lib.nvq_status_string(status).decode()
        if status == NVQ_ERR_CUDA:
            msg += f" [{_lib.nvq_last_cuda_error().decode()}]"
        super().__init__(f"{func}: status {status}: {msg}")


def lib() -> ctypes.CDLL:
    """The loaded ``libnvq.so`` (raw C entry points)."""
    return _lib


def _check(func: str, status: int) -> None:
    if status != NVQ_OK:
        raise NVQError(func, status)


def _ptr(t) -> int:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return int(t)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def version() -> int:
    return _lib.nvq_version()


# ---------------------------------------------------------------------------

def pack_nvfp4(w: np.ndarray):
    """Host NVFP4 packer: fp32 W[N, K] -> (codes uint8 [N, K/2], scales uint8
    [N, K/16], g float)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 16), np.uint8)
    g = ctypes.c_float(0.0)
    _check("nvq_pack_nvfp4", _lib.nvq_pack_nvfp4(
        _ptr(w), N, K, _ptr(codes), _ptr(scales), ctypes.addressof(g)))
    return codes, scales, g.value


def quantize_act_q8_0(x: torch.Tensor, q: torch.Tensor | None = None,
                      d: torch.Tensor | None = None, stream=None):
    """Q8_0 of device fp32 x[M, K] -> (q int8 [M, K], d float16 [M, K/32])."""
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if d is None:
        d = torch.empty((M, K // 32), dtype=torch.float16, device=x.device)
    _check("nvq_quantize_act_q8_0", _lib.nvq_quantize_act_q8_0(
        _ptr(x), M, K, _ptr(q), _ptr(d), _stream(stream)))
    return q, d


def gemv(codes: torch.Tensor, scales: torch.Tensor, g: float, q: torch.Tensor,
         d: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode GEMV (M = 1..16): y[M, N] fp32."""
    N = codes.shape[0]
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=q.device)
    _check("nvq_gemv", _lib.nvq_gemv(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(q), _ptr(d), M, _ptr(y),
        _stream(stream)))
    return y


def gemv_requant(codes: torch.Tensor, scales: torch.Tensor, g: float, q: torch.Tensor,
                 d: torch.Tensor, counters: torch.Tensor, y: torch.Tensor | None = None,
                 q_out: torch.Tensor | None = None, d_out: torch.Tensor | None = None,
                 stream=None):
    """One token's GEMV that also emits Q8_0 of y (nvq_gemv_requant):
    returns (y fp32 [1, N], q_out int8 [1, N], d_out float16 [1, N/32]).
    counters: device int32 [N/32], zero before the first call."""
    N = codes.shape[0]
    M, K = q.shape
    if y is None:
        y = torch.empty((1, N), dtype=torch.float32, device=q.device)
    if q_out is None:
        q_out = torch.empty((1, N), dtype=torch.int8, device=q.device)
    if d_out is None:
        d_out = torch.empty((1, N // 32), dtype=torch.float16, device=q.device)
    _check("nvq_gemv_requant", _lib.nvq_gemv_requant(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(q), _ptr(d), _ptr(y), _ptr(q_out),
        _ptr(d_out), _ptr(counters), _stream(stream)))
    return y, q_out, d_out


def gemv_grouped(mats, q: torch.Tensor, d: torch.Tensor, ys=None, stream=None):
    """nvq_gemv of several (codes, scales, g) with the same K against one
    activation: returns the list of y [M, N_i]."""
    M, K = q.shape
    arr = (Linear * len(mats))()
    for i, (codes, scales, g) in enumerate(mats):
        arr[i] = Linear(codes.data_ptr(), scales.data_ptr(), float(g), codes.shape[0],
                        codes.shape[1] * 2)
    if ys is None:
        ys = [torch.empty((M, c.shape[0]), dtype=torch.float32, device=q.device)
              for c, _, _ in mats]
    ptrs = (_vp * len(mats))(*[t.data_ptr() for t in ys])
    _check("nvq_gemv_grouped", _lib.nvq_gemv_grouped(arr, len(mats), _ptr(q), _ptr(d), M, ptrs,
                                                     _stream(stream)))
    return ys


def moe_gemv(codes: torch.Tensor, scales: torch.Tensor, g: torch.Tensor, ids: torch.Tensor,
             q: torch.Tensor, d: torch.Tensor, y: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """Mixture-of-experts decode GEMV (nvq_moe_gemv): codes [E, N, K/2],
    scales [E, N, K/16], g float32 [E], ids int32 [T, top_k] (all on the
    device); returns y fp32 [T, top_k, N]."""
    E, N = codes.shape[0], codes.shape[1]
    T, K = q.shape
    top_k = ids.shape[1]
    if y is None:
        y = torch.empty((T, top_k, N), dtype=torch.float32, device=q.device)
    _check("nvq_moe_gemv", _lib.nvq_moe_gemv(
        _ptr(codes), _ptr(scales), _ptr(g), E, N, K, _ptr(ids), T, top_k, _ptr(q), _ptr(d),
        _ptr(y), _stream(stream)))
    return y


def gemm_w4a16(codes: torch.Tensor, scales: torch.Tensor, g: float, x: torch.Tensor,
               y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """NVFP4 weights x fp16 activations (nvq_gemm_w4a16): x float16 [M, K]
    on the device, M = 1..16; returns y fp32 [M, N]."""
    N = codes.shape[0]
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    nbytes = int(_lib.nvq_gemm_w4a16_workspace_size(M, N, K))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    _check("nvq_gemm_w4a16", _lib.nvq_gemm_w4a16(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(x), M, _ptr(y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return y


def quantize_act_nvfp4(x: torch.Tensor, stream=None):
    """NVFP4 activations (nvq_quantize_act_nvfp4): x float32 [M, K] on the
    device; returns (codes uint8 [M, K/2], scales uint8 [M, K/16], g float32 [M])."""
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    g = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("nvq_quantize_act_nvfp4", _lib.nvq_quantize_act_nvfp4(
        _ptr(x), M, K, _ptr(codes), _ptr(scales), _ptr(g), _stream(stream)))
    return codes, scales, g


def gemm_nvf4(w_codes: torch.Tensor, w_scales: torch.Tensor, g_w: float, a_codes: torch.Tensor,
              a_scales: torch.Tensor, a_g: torch.Tensor, y: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """NVFP4 weights x NVFP4 activations (nvq_gemm_nvf4) on the block-scaled
    FP4 tensor-core path; returns y fp32 [M, N]."""
    N = w_codes.shape[0]
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=a_codes.device)
    _check("nvq_gemm_nvf4", _lib.nvq_gemm_nvf4(
        _ptr(w_codes), _ptr(w_scales), float(g_w), N, K, _ptr(a_codes), _ptr(a_scales),
        _ptr(a_g), M, _ptr(y), _stream(stream)))
    return y


def gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.nvq_gemm_workspace_size(M, N, K))


def gemm(codes: torch.Tensor, scales: torch.Tensor, g: float, q: torch.Tensor,
         d: torch.Tensor, y: torch.Tensor | None = None,
         workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill GEMM (tcgen05): y[M, N] fp32."""
    N = codes.shape[0]
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=q.device)
    ws_bytes = gemm_workspace_size(M, N, K)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    _check("nvq_gemm", _lib.nvq_gemm(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(q), _ptr(d), M, _ptr(y),
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return y


def gemm_noalloc(codes: torch.Tensor, scales: torch.Tensor, g: float, q: torch.Tensor,
                 d: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill GEMM with the library's own 64 MiB device scratch instead of a
    caller workspace (nvq_gemm_noalloc): y[M, N] fp32."""
    N = codes.shape[0]
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=q.device)
    _check("nvq_gemm_noalloc", _lib.nvq_gemm_noalloc(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(q), _ptr(d), M, _ptr(y),
        _stream(stream)))
    return y


def debug_subblock_sums(codes: torch.Tensor, scales: torch.Tensor, g: float, q: torch.Tensor,
                        d: torch.Tensor, y: torch.Tensor | None = None,
                        isum: torch.Tensor | None = None, stream=None):
    """nvq_gemv that also exports its integer per-16 subblock sums:
    returns (y fp32 [M, N], isum int32 [M, N, K/16])."""
    N = codes.shape[0]
    M, K = q.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=q.device)
    if isum is None:
        isum = torch.empty((M, N, K // 16), dtype=torch.int32, device=q.device)
    _check("nvq_debug_subblock_sums", _lib.nvq_debug_subblock_sums(
        _ptr(codes), _ptr(scales), float(g), N, K, _ptr(q), _ptr(d), M, _ptr(y), _ptr(isum),
        _stream(stream)))
    return y, isum


FLAG_GEMV_TIMEOUT = 1
FLAG_GEMM_TIMEOUT = 2
FLAG_BAD_INDEX = 4


def error_flags(clear: bool = False) -> int:
    """Device-side error flags of the current device (NVQ_FLAG_* bits);
    synchronous.  Read them after synchronising the streams used."""
    v = ctypes.c_uint(0)
    _check("nvq_error_flags", _lib.nvq_error_flags(ctypes.byref(v), 1 if clear else 0))
    return int(v.value)


def debug_stalled_wait(limit_ns: int, result: torch.Tensor, stream=None) -> None:
    """Test-only: one bounded pipeline wait that can never complete
    (nvq_debug_stalled_wait); result is a device int32 [2] tensor."""
    _check("nvq_debug_stalled_wait", _lib.nvq_debug_stalled_wait(
        int(limit_ns), _ptr(result), _stream(stream)))


class DecoderStack:
    """Device-resident linear layers of a dense decoder stack (7 NVFP4
    matrices per layer: q, k, v, o, up, gate, down) and the buffers of one
    pass; ``forward`` enqueues every layer through ``nvq_decoder_stack``."""

    def __init__(self, layers, M: int, device="cuda"):
        """layers: list of n_layers lists of 7 (codes, scales, g) with codes
        and scales device tensors."""
        self.n_layers = len(layers)
        self.M = M
        arr = (Linear * (STACK_LINEARS * self.n_layers))()
        self._keep = []
        for l, layer in enumerate(layers):
            if len(layer) != STACK_LINEARS:
                raise ValueError("each layer needs 7 matrices")
            for i, (codes, scales, g) in enumerate(layer):
                arr[STACK_LINEARS * l + i] = Linear(codes.data_ptr(), scales.data_ptr(), float(g),
                                                    codes.shape[0], codes.shape[1] * 2)
                self._keep.append((codes, scales))
        self.linears = arr
        self.outs = [torch.empty((M, layers[0][i][0].shape[0]), dtype=torch.float32, device=device)
                     for i in range(STACK_LINEARS)]
        self._outs_ptrs = (_vp * STACK_LINEARS)(*[t.data_ptr() for t in self.outs])
        nbytes = int(_lib.nvq_decoder_stack_workspace_size(arr, M))
        if nbytes == 0:
            raise NVQError("nvq_decoder_stack_workspace_size", NVQ_ERR_BAD_SHAPE)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def forward(self, x: torch.Tensor, stream=None, n_layers: int | None = None):
        n = self.n_layers if n_layers is None else n_layers
        _check("nvq_decoder_stack", _lib.nvq_decoder_stack(
            self.linears, n, _ptr(x), self.M, self._outs_ptrs, _ptr(self.workspace),
            self.workspace.numel(), _stream(stream)))
        return self.outs
