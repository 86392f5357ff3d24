"""Python binding of ``libspear.so``: the B200 W4 linear layer with a per-token-gated
low-rank error compensator (SPEAR: Post-Quantization Error-Adaptive Recovery,
technical summary section 2.1A).

Argument marshalling only.  Every step of the layer runs in the library's CUDA
kernels; PyTorch supplies device memory and streams.  The names match the C ABI
in ``include/spear.h``.  There is no CPU fallback: if the library is missing or
fails to load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspear.so")

SPEAR_OK = 0
(SPEAR_ERR_INVALID_ARG, SPEAR_ERR_UNSUPPORTED_SHAPE, SPEAR_ERR_MISALIGNED, SPEAR_ERR_WORKSPACE_TOO_SMALL,
 SPEAR_ERR_CUDA, SPEAR_ERR_TIMEOUT) = 1, 2, 3, 4, 5, 6
SPEAR_BF16, SPEAR_FP32 = 0, 1
SPEAR_KERNEL_AUTO, SPEAR_KERNEL_SPLITK, SPEAR_KERNEL_TC05, SPEAR_KERNEL_STREAM, SPEAR_KERNEL_STREAM_RK = 0, 1, 2, 3, 4
SPEAR_PLAN_SEPARATE_EC, SPEAR_PLAN_DEEP_RING, SPEAR_PLAN_W4_TILES = 1, 2, 4
SPEAR_W4_ROWS, SPEAR_W4_TILES = 1, 2
STATUS_NAMES = {0: "SPEAR_OK", 1: "SPEAR_ERR_INVALID_ARG", 2: "SPEAR_ERR_UNSUPPORTED_SHAPE",
                3: "SPEAR_ERR_MISALIGNED", 4: "SPEAR_ERR_WORKSPACE_TOO_SMALL", 5: "SPEAR_ERR_CUDA",
                6: "SPEAR_ERR_TIMEOUT"}
EXPORTED = ["spear_pack_w4", "spear_debug_unpack_w4", "spear_tile_w4", "spear_gemm_plan", "spear_gemm_plan_tiled",
            "spear_gemm_plan_formats",
            "spear_plan_update", "spear_w4ec_gemm",
            "spear_w4ec_gemm_noalloc", "spear_noalloc_get_device_status", "spear_get_device_status", "spear_status_string", "spear_version",
            "spear_latency_table", "spear_predict_step_us", "spear_pick_prefill_chunk",
            "spear_pack_w4_grouped", "spear_grouped_workspace_bytes", "spear_w4ec_gemm_grouped"]


class SpearError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({spear_status_string(status)})")


class spear_plan(ctypes.Structure):
    _fields_ = [("kernel_id", ctypes.c_int32), ("tile_n", ctypes.c_int32), ("split_k", ctypes.c_int32),
                ("tile_m", ctypes.c_int32), ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_size_t)]

    def __repr__(self):
        return (f"spear_plan(kernel_id={self.kernel_id}, tile_n={self.tile_n}, split_k={self.split_k}, "
                f"tile_m={self.tile_m}, flags={self.flags}, workspace_bytes={self.workspace_bytes})")


class spear_linear_desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("rank", ctypes.c_int32), ("count", ctypes.c_int32)]


class spear_latency_entry(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("has_ec", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("us", ctypes.c_double)]


class spear_ec(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("w_g", ctypes.c_void_p),
                ("b_g", ctypes.c_float), ("rank", ctypes.c_int32),
                ("gate_w1", ctypes.c_void_p), ("gate_b1", ctypes.c_void_p), ("gate_w2", ctypes.c_void_p),
                ("gate_b2", ctypes.c_void_p), ("gate_hidden", ctypes.c_int32), ("alpha", ctypes.c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python w4_gemm_error_channel_b200/build.py` "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.spear_pack_w4.argtypes = [P, ctypes.c_int, I64, I64, P, P, P, P]
    lib.spear_debug_unpack_w4.argtypes = [P, P, I64, I64, P, P, P]
    lib.spear_tile_w4.argtypes = [P, I64, I64, P, P]
    lib.spear_gemm_plan.argtypes = [I64, I64, I64, ctypes.c_int32, ctypes.c_int, ctypes.POINTER(spear_plan)]
    lib.spear_gemm_plan_tiled.argtypes = [I64, I64, I64, ctypes.c_int32, ctypes.c_int, ctypes.POINTER(spear_plan)]
    lib.spear_gemm_plan_formats.argtypes = [I64, I64, I64, ctypes.c_int32, ctypes.c_int, ctypes.c_int32,
                                            ctypes.POINTER(spear_plan)]
    lib.spear_plan_update.argtypes = [ctypes.POINTER(spear_plan), I64, I64, I64, ctypes.c_int32]
    lib.spear_w4ec_gemm.argtypes = [ctypes.POINTER(spear_plan), P, I64, I64, I64, P, P, P,
                                    ctypes.POINTER(spear_ec), P, ctypes.c_int, P, ctypes.c_size_t, P]
    lib.spear_w4ec_gemm_noalloc.argtypes = [ctypes.POINTER(spear_plan), P, I64, I64, I64, P, P, P,
                                            ctypes.POINTER(spear_ec), P, ctypes.c_int, P]
    lib.spear_get_device_status.argtypes = [P, ctypes.c_int, P]
    lib.spear_noalloc_get_device_status.argtypes = [ctypes.c_int, P]
    lib.spear_pack_w4_grouped.argtypes = [P, ctypes.c_int, I64, I64, I64, P, P, P, P]
    lib.spear_grouped_workspace_bytes.argtypes = [I64, I64, I64, I64, ctypes.c_int32,
                                                  ctypes.POINTER(ctypes.c_size_t)]
    lib.spear_w4ec_gemm_grouped.argtypes = [P, I64, I64, I64, I64, P, P, P, ctypes.POINTER(spear_ec), P,
                                            ctypes.c_int, P, ctypes.c_size_t, P]
    LD, LE = ctypes.POINTER(spear_linear_desc), ctypes.POINTER(spear_latency_entry)
    lib.spear_latency_table.argtypes = [LE, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    lib.spear_predict_step_us.argtypes = [LD, ctypes.c_int32, I64, ctypes.c_double, LE, ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_double)]
    lib.spear_pick_prefill_chunk.argtypes = [LD, ctypes.c_int32, I64, I64, I64, ctypes.c_double, ctypes.c_double,
                                             LE, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64),
                                             ctypes.POINTER(ctypes.c_double)]
    lib.spear_status_string.argtypes = [ctypes.c_int]
    lib.spear_status_string.restype = ctypes.c_char_p
    lib.spear_version.restype = ctypes.c_int
    for fn in ("spear_pack_w4", "spear_debug_unpack_w4", "spear_gemm_plan", "spear_plan_update", "spear_w4ec_gemm",
               "spear_w4ec_gemm_noalloc", "spear_noalloc_get_device_status", "spear_get_device_status",
               "spear_latency_table",
               "spear_predict_step_us", "spear_pick_prefill_chunk", "spear_pack_w4_grouped",
               "spear_grouped_workspace_bytes", "spear_w4ec_gemm_grouped"):
        getattr(lib, fn).restype = ctypes.c_int
    return lib


_lib = _load()


def _check(fn: str, status: int):
    if status != SPEAR_OK:
        raise SpearError(fn, status)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def spear_status_string(status: int) -> str:
    return _lib.spear_status_string(int(status)).decode()


def spear_version() -> int:
    return int(_lib.spear_version())


@dataclasses.dataclass
class EC:
    """One layer's error compensator: A bf16 [K,r], B bf16 [r,N], w_g bf16 [K], b_g float.

    Optional bottleneck-MLP gate (the pages' gamma): gate_w1 fp32 [H,r], gate_b1 [H], gate_w2 [r,H],
    gate_b2 [r] and alpha; with it, u = alpha * sigmoid(W2 relu(W1 t + b1) + b2) * t and the scalar
    gate (w_g, b_g) does not enter the result.
    """
    A: torch.Tensor
    B: torch.Tensor
    w_g: torch.Tensor
    b_g: float = 0.0
    gate_w1: Optional[torch.Tensor] = None
    gate_b1: Optional[torch.Tensor] = None
    gate_w2: Optional[torch.Tensor] = None
    gate_b2: Optional[torch.Tensor] = None
    alpha: float = 1.0

    @property
    def rank(self) -> int:
        return int(self.A.shape[1])

    def as_c(self) -> spear_ec:
        for name in ("A", "B", "w_g"):
            t = getattr(self, name)
            _dev(t, name)
            if t.dtype != torch.bfloat16:
                raise ValueError(f"EC.{name} must be bf16")
        c = spear_ec(self.A.data_ptr(), self.B.data_ptr(), self.w_g.data_ptr(), float(self.b_g), self.rank)
        if self.gate_w1 is not None:
            for name in ("gate_w1", "gate_b1", "gate_w2", "gate_b2"):
                t = getattr(self, name)
                if t is None:
                    raise ValueError(f"EC.{name} is required with the MLP gate")
                _dev(t, name)
                if t.dtype != torch.float32:
                    raise ValueError(f"EC.{name} must be fp32")
            c.gate_w1, c.gate_b1 = self.gate_w1.data_ptr(), self.gate_b1.data_ptr()
            c.gate_w2, c.gate_b2 = self.gate_w2.data_ptr(), self.gate_b2.data_ptr()
            c.gate_hidden, c.alpha = int(self.gate_w1.shape[0]), float(self.alpha)
        return c


def spear_pack_w4(W: torch.Tensor, packed=None, scale=None, zero=None, stream=None):
    """RTN per-channel int4 packing of W [N,K] (fp32 or bf16) -> (packed u8 [N,K/2], scale f16 [N], zero f16 [N])."""
    _dev(W, "W")
    N, K = W.shape
    if W.dtype == torch.float32:
        wd = SPEAR_FP32
    elif W.dtype == torch.bfloat16:
        wd = SPEAR_BF16
    else:
        raise ValueError("W must be fp32 or bf16")
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device) if packed is None else packed
    scale = torch.empty(N, dtype=torch.float16, device=W.device) if scale is None else scale
    zero = torch.empty(N, dtype=torch.float16, device=W.device) if zero is None else zero
    _check("spear_pack_w4", _lib.spear_pack_w4(_p(W), wd, N, K, _p(packed), _p(scale), _p(zero), _stream(stream)))
    return packed, scale, zero


def spear_debug_unpack_w4(packed: torch.Tensor, zero: torch.Tensor, K: int, want_q=True, want_qz=True,
                          stream=None):
    """Test hook: (q u8 [N,K] or None, (q - z) bf16 [N,K] or None)."""
    _dev(packed, "packed")
    N = packed.shape[0]
    q = torch.empty((N, K), dtype=torch.uint8, device=packed.device) if want_q else None
    qz = torch.empty((N, K), dtype=torch.bfloat16, device=packed.device) if want_qz else None
    _check("spear_debug_unpack_w4",
           _lib.spear_debug_unpack_w4(_p(packed), _p(zero), N, K, _p(q), _p(qz), _stream(stream)))
    return q, qz


def spear_gemm_plan(M: int, N: int, K: int, rank: int = 0, device: int = -1) -> spear_plan:
    plan = spear_plan()
    _check("spear_gemm_plan", _lib.spear_gemm_plan(M, N, K, rank, device, ctypes.byref(plan)))
    return plan


def spear_gemm_plan_tiled(M: int, N: int, K: int, rank: int = 0, device: int = -1) -> spear_plan:
    """Plan for codes in spear_tile_w4's tile order (the register-path stream kernel, M <= 64)."""
    plan = spear_plan()
    _check("spear_gemm_plan_tiled", _lib.spear_gemm_plan_tiled(M, N, K, rank, device, ctypes.byref(plan)))
    return plan


def spear_gemm_plan_formats(M: int, N: int, K: int, rank: int = 0, formats: int = SPEAR_W4_ROWS | SPEAR_W4_TILES,
                            device: int = -1) -> spear_plan:
    """Plan among the code orders held (SPEAR_W4_ROWS, SPEAR_W4_TILES): the tile order where it was
    measured faster for this shape."""
    plan = spear_plan()
    _check("spear_gemm_plan_formats", _lib.spear_gemm_plan_formats(M, N, K, rank, device, formats, ctypes.byref(plan)))
    return plan


def spear_tile_w4(packed: torch.Tensor, tiled=None, stream=None) -> torch.Tensor:
    """Codes of spear_pack_w4 (u8 [N, K/2]) in the tile order of the register-path stream kernel
    (u8 [N, K/2] storage holding the reordered bytes)."""
    _dev(packed, "packed")
    N, half = packed.shape
    tiled = torch.empty_like(packed) if tiled is None else tiled
    _check("spear_tile_w4", _lib.spear_tile_w4(_p(packed), N, 2 * half, _p(tiled), _stream(stream)))
    return tiled


def spear_plan_update(plan: spear_plan, M: int, N: int, K: int, rank: int = 0) -> spear_plan:
    """Checks a plan whose fields were changed and recomputes its workspace_bytes (in place)."""
    _check("spear_plan_update", _lib.spear_plan_update(ctypes.byref(plan), M, N, K, rank))
    return plan


def spear_pack_w4_grouped(W: torch.Tensor, group: int, stream=None):
    """Group-wise RTN W4 packing of W [N, K] (fp32 or bf16, on the GPU): packed [N, K/2] uint8,
    scale and zero [N, K/group] fp16."""
    _dev(W, "W")
    if W.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("W must be fp32 or bf16")
    W = W.contiguous()
    N, K = W.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scale = torch.empty((N, max(K // max(group, 1), 1)), dtype=torch.float16, device=W.device)
    zero = torch.empty_like(scale)
    dt = SPEAR_BF16 if W.dtype == torch.bfloat16 else SPEAR_FP32
    _check("spear_pack_w4_grouped", _lib.spear_pack_w4_grouped(_p(W), dt, N, K, group, _p(packed), _p(scale),
                                                              _p(zero), _stream(stream)))
    return packed, scale, zero


def spear_grouped_workspace_bytes(M: int, N: int, K: int, group: int, rank: int = 0) -> int:
    out = ctypes.c_size_t()
    _check("spear_grouped_workspace_bytes", _lib.spear_grouped_workspace_bytes(M, N, K, group, rank, ctypes.byref(out)))
    return out.value


def spear_w4ec_gemm_grouped(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                            group: int, ec: Optional[EC] = None, y: Optional[torch.Tensor] = None,
                            y_dtype=torch.bfloat16, workspace: Optional[torch.Tensor] = None, stream=None):
    """y = x What^T + g(x) (x A) B with group-wise scales (scale, zero [N, K/group])."""
    _dev(x, "x")
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    M, K = x.shape
    N = packed.shape[0]
    rank = ec.rank if ec is not None else 0
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    yd = SPEAR_FP32 if y.dtype == torch.float32 else SPEAR_BF16
    if workspace is None:
        workspace = alloc_workspace(spear_grouped_workspace_bytes(M, N, K, group, rank), x.device)
    ec_c = ctypes.byref(ec.as_c()) if ec is not None else None
    _check("spear_w4ec_gemm_grouped",
           _lib.spear_w4ec_gemm_grouped(_p(x), M, N, K, group, _p(packed), _p(scale), _p(zero), ec_c, _p(y), yd,
                                        _p(workspace), workspace.numel(), _stream(stream)))
    return y


def _linears(linears):
    """(N, K, rank, count) tuples -> a ctypes array of spear_linear_desc."""
    arr = (spear_linear_desc * len(linears))()
    for i, (N, K, rank, count) in enumerate(linears):
        arr[i].N, arr[i].K, arr[i].rank, arr[i].count = N, K, rank, count
    return arr


def _lut(lut):
    """None (the built-in table) or (M, N, K, has_ec, us) tuples -> (pointer, length)."""
    if lut is None:
        return None, 0
    arr = (spear_latency_entry * len(lut))()
    for i, (M, N, K, has_ec, us) in enumerate(lut):
        arr[i].M, arr[i].N, arr[i].K, arr[i].has_ec, arr[i].us = M, N, K, int(bool(has_ec)), us
    return arr, len(lut)


def spear_latency_table():
    """The built-in kernel-latency table as (M, N, K, has_ec, us) tuples."""
    n = ctypes.c_int32()
    _check("spear_latency_table", _lib.spear_latency_table(None, 0, ctypes.byref(n)))
    arr = (spear_latency_entry * n.value)()
    _check("spear_latency_table", _lib.spear_latency_table(arr, n.value, ctypes.byref(n)))
    return [(e.M, e.N, e.K, e.has_ec, e.us) for e in arr]


def spear_predict_step_us(linears, M: int, fixed_us: float = 0.0, lut=None) -> float:
    """Predicted latency (us) of one step that runs every (N, K, rank, count) linear on M tokens."""
    la, (lp, ln) = _linears(linears), _lut(lut)
    out = ctypes.c_double()
    _check("spear_predict_step_us",
           _lib.spear_predict_step_us(la, len(linears), M, fixed_us, lp, ln, ctypes.byref(out)))
    return out.value


def spear_pick_prefill_chunk(linears, decode_tokens: int, max_chunk: int, slo_us: float, granule: int = 128,
                             fixed_us: float = 0.0, lut=None):
    """(chunk, predicted_us): the largest prefill chunk (a multiple of granule) whose step with
    decode_tokens + chunk tokens is predicted to meet slo_us."""
    la, (lp, ln) = _linears(linears), _lut(lut)
    chunk, pred = ctypes.c_int64(), ctypes.c_double()
    _check("spear_pick_prefill_chunk",
           _lib.spear_pick_prefill_chunk(la, len(linears), decode_tokens, max_chunk, granule, slo_us, fixed_us,
                                         lp, ln, ctypes.byref(chunk), ctypes.byref(pred)))
    return chunk.value, pred.value


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled workspace (the control words must start at zero)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8,
                       device=device if device is not None else torch.cuda.current_device())


def spear_w4ec_gemm(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                    ec: Optional[EC] = None, y: Optional[torch.Tensor] = None, y_dtype=torch.bfloat16,
                    workspace: Optional[torch.Tensor] = None, plan: Optional[spear_plan] = None, stream=None):
    """y = x dequant(Wq)^T + g(x) (x A) B.  Returns y [M,N] (bf16, or fp32 for checks)."""
    _dev(x, "x")
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    M, K = x.shape
    N = packed.shape[0]
    rank = ec.rank if ec is not None else 0
    if plan is None:
        plan = spear_gemm_plan(M, N, K, rank, x.device.index)
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    yd = SPEAR_FP32 if y.dtype == torch.float32 else SPEAR_BF16
    if workspace is None:
        workspace = alloc_workspace(plan.workspace_bytes, x.device)
    ec_c = ctypes.byref(ec.as_c()) if ec is not None else None
    _check("spear_w4ec_gemm",
           _lib.spear_w4ec_gemm(ctypes.byref(plan), _p(x), M, N, K, _p(packed), _p(scale), _p(zero), ec_c,
                                _p(y), yd, _p(workspace), workspace.numel(), _stream(stream)))
    return y


def spear_w4ec_gemm_noalloc(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                            y: torch.Tensor, ec: Optional[EC] = None, plan: Optional[spear_plan] = None,
                            stream=None):
    """The layer for up to 64 tokens with the library's own device scratch (no workspace).

    For callers that cannot allocate device memory: y [M, N] (bf16, or fp32 for checks) is the
    caller's, and neither this wrapper nor the C call allocates anything.  Calls sharing the
    library's scratch must not overlap on the GPU.
    """
    _dev(x, "x")
    _dev(y, "y")
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    M, K = x.shape
    N = packed.shape[0]
    if y.dtype not in (torch.bfloat16, torch.float32) or tuple(y.shape) != (M, N):
        raise ValueError("y must be a contiguous bf16 or fp32 [M, N] tensor")
    yd = SPEAR_FP32 if y.dtype == torch.float32 else SPEAR_BF16
    ec_c = ctypes.byref(ec.as_c()) if ec is not None else None
    plan_c = ctypes.byref(plan) if plan is not None else None
    _check("spear_w4ec_gemm_noalloc",
           _lib.spear_w4ec_gemm_noalloc(plan_c, _p(x), M, N, K, _p(packed), _p(scale), _p(zero), ec_c, _p(y), yd,
                                        _stream(stream)))
    return y


class W4ECLayer:
    """One quantised layer bound once, called many times: y = x dequant(Wq)^T + g(x) (x A) B.

    Checks and converts the weight-side arguments (packed weights, scales, zero-points and the
    compensator) once, keeps one workspace and a plan per batch size, so that a call marshals
    only x, y and the stream into one spear_w4ec_gemm call.  The tensors must stay alive and
    unchanged while the layer is used.  Calls that share the layer's workspace must be ordered
    on one stream; the first call with a new batch size may replace the workspace by a larger
    one (plan() every size up front to avoid that).
    """

    def __init__(self, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, ec: Optional[EC] = None,
                 y_dtype=torch.bfloat16, tiled: Optional[torch.Tensor] = None):
        for name, t in (("packed", packed), ("scale", scale), ("zero", zero)):
            _dev(t, name)
        if tiled is not None:
            _dev(tiled, "tiled")
            if tiled.numel() != packed.numel():
                raise ValueError("tiled must hold the same codes as packed (spear_tile_w4(packed))")
        self.N, self.K = int(packed.shape[0]), int(packed.shape[1]) * 2
        self.device = packed.device
        self._index = packed.get_device()
        self.y_dtype = y_dtype
        self._yd = SPEAR_FP32 if y_dtype == torch.float32 else SPEAR_BF16
        self.rank = ec.rank if ec is not None else 0
        self._keep = (packed, scale, zero, ec, tiled)
        self._ec_c = ec.as_c() if ec is not None else None
        self._ec_ref = ctypes.byref(self._ec_c) if ec is not None else None
        self._w = (packed.data_ptr(), scale.data_ptr(), zero.data_ptr())
        # The tile order serves the scalar gate only.
        self._tiled = tiled.data_ptr() if tiled is not None and (ec is None or ec.gate_w1 is None) else None
        self._plans = {}
        self._ws = None

    def plan(self, M: int) -> spear_plan:
        p = self._plans.get(M)
        if p is None:
            if self._tiled is not None:
                p = spear_gemm_plan_formats(M, self.N, self.K, self.rank, SPEAR_W4_ROWS | SPEAR_W4_TILES,
                                            self.device.index)
            else:
                p = spear_gemm_plan(M, self.N, self.K, self.rank, self.device.index)
            if self._ws is None or self._ws.numel() < p.workspace_bytes:
                self._ws = alloc_workspace(p.workspace_bytes, self.device)
            self._plans[M] = (p, ctypes.byref(p))
            return p
        return p[0]

    @property
    def workspace(self) -> torch.Tensor:
        return self._ws

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        M = int(x.shape[0])
        entry = self._plans.get(M)
        if entry is None:
            self.plan(M)
            entry = self._plans[M]
        if (x.dtype != torch.bfloat16 or x.get_device() != self._index or not x.is_contiguous()
                or x.dim() != 2 or x.shape[1] != self.K):
            raise ValueError("x must be a contiguous bf16 [M, K] tensor on the layer's device")
        if y is None:
            y = torch.empty((M, self.N), dtype=self.y_dtype, device=self.device)
        elif (y.dtype != self.y_dtype or y.get_device() != self._index or not y.is_contiguous()
              or tuple(y.shape) != (M, self.N)):
            raise ValueError("y must be a contiguous [M, N] tensor of the layer's output dtype on its device")
        sh = stream.cuda_stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        ws = self._ws
        codes = self._tiled if entry[0].flags & SPEAR_PLAN_W4_TILES else self._w[0]
        st = _lib.spear_w4ec_gemm(entry[1], x.data_ptr(), M, self.N, self.K, codes, self._w[1], self._w[2],
                                  self._ec_ref, y.data_ptr(), self._yd, ws.data_ptr(), ws.numel(), sh)
        if st != SPEAR_OK:
            raise SpearError("spear_w4ec_gemm", st)
        return y


def spear_get_device_status(workspace: torch.Tensor, clear: bool = True, stream=None) -> int:
    return int(_lib.spear_get_device_status(_p(workspace), int(clear), _stream(stream)))


def spear_noalloc_get_device_status(clear: bool = True, stream=None) -> int:
    """Error word of spear_w4ec_gemm_noalloc's library-owned array (SPEAR_OK or SPEAR_ERR_TIMEOUT)."""
    return int(_lib.spear_noalloc_get_device_status(int(clear), _stream(stream)))


def loaded_library_path() -> str:
    return LIB_PATH
