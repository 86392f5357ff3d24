"""CPU oracle for the W4 + per-token-gated error-compensator linear layer.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package.  The CUDA library never uses
it, and it shares no code with the CUDA library.

The arithmetic lives in ``spear_oracle.c`` (plain C, fp64 after quantisation);
this module compiles it with gcc and wraps it with ctypes.  Every function cites
the passage it follows in the C source's header: the SPEAR technical summary,
section 2.1A (input-adaptive error compensators with a per-token gate) and
section 3.1 (RTN per-channel 4-bit weights).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spear_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-Wall", "-Wextra", "-Wno-unused-parameter"]

_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile an oracle source into a shared library (gcc, no CUDA)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", *_CFLAGS, src, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """ctypes wrapper around one build of ``spear_oracle.c``."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_quantize_rtn.argtypes = [P, I64, I64, P, P, P]
        lib.oracle_pack_nibbles.argtypes = [P, I64, I64, P]
        lib.oracle_unpack_nibbles.argtypes = [P, I64, I64, P]
        lib.oracle_pack_w4.argtypes = [P, I64, I64, P, P, P]
        lib.oracle_dequant_w4.argtypes = [P, P, P, I64, I64, P]
        lib.oracle_ec_gate.argtypes = [P, I64, I64, P, ctypes.c_int32, P, ctypes.c_float, P, P, P]
        lib.oracle_w4ec_gemm.argtypes = [P, I64, I64, I64, P, P, P, P, P, P, ctypes.c_float,
                                         ctypes.c_int32, P]
        lib.oracle_w4ec_gemm_sampled.argtypes = [P, I64, I64, I64, P, P, P, P, P, P, ctypes.c_float,
                                                 ctypes.c_int32, P, P, I64, P]
        lib.oracle_w4ec_gemm_grouped.argtypes = [P, I64, I64, I64, I64, P, P, P, P, P, P, ctypes.c_float,
                                                 ctypes.c_int32, P]
        lib.oracle_w4ec_gemm_mlp.argtypes = [P, I64, I64, I64, P, P, P, P, P, ctypes.c_int32, P, P, P, P,
                                             ctypes.c_int32, ctypes.c_float, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        self._lib = lib
        self.path = lib_path

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def f32_to_f16_bits(self, v: float) -> int:
        """IEEE binary16 encoding of an fp32 value, round to nearest even."""
        return int(self._lib.oracle_f32_to_f16(ctypes.c_float(v)))

    def f16_bits_to_f64(self, b: int) -> float:
        return float(self._lib.oracle_f16_to_f64(ctypes.c_uint16(b)))

    def quantize_rtn(self, W: np.ndarray):
        """RTN per-channel asymmetric W4: W fp32 [N,K] -> (q u8 [N,K], s bits u16 [N], z bits u16 [N])."""
        W = _c(W, np.float32)
        N, K = W.shape
        q = np.empty((N, K), np.uint8)
        s = np.empty(N, np.uint16)
        z = np.empty(N, np.uint16)
        self._lib.oracle_quantize_rtn(_ptr(W), N, K, _ptr(q), _ptr(s), _ptr(z))
        return q, s, z

    def pack_nibbles(self, q: np.ndarray) -> np.ndarray:
        q = _c(q, np.uint8)
        N, K = q.shape
        out = np.empty((N, K // 2), np.uint8)
        self._lib.oracle_pack_nibbles(_ptr(q), N, K, _ptr(out))
        return out

    def unpack_nibbles(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = _c(packed, np.uint8)
        N = packed.shape[0]
        out = np.empty((N, K), np.uint8)
        self._lib.oracle_unpack_nibbles(_ptr(packed), N, K, _ptr(out))
        return out

    def pack_w4(self, W: np.ndarray):
        """W fp32 [N,K] -> (packed u8 [N,K/2], s bits u16 [N], z bits u16 [N])."""
        W = _c(W, np.float32)
        N, K = W.shape
        packed = np.empty((N, K // 2), np.uint8)
        s = np.empty(N, np.uint16)
        z = np.empty(N, np.uint16)
        self._lib.oracle_pack_w4(_ptr(W), N, K, _ptr(packed), _ptr(s), _ptr(z))
        return packed, s, z

    def dequant_w4(self, packed, s_bits, z_bits, K: int) -> np.ndarray:
        packed = _c(packed, np.uint8)
        N = packed.shape[0]
        out = np.empty((N, K), np.float64)
        self._lib.oracle_dequant_w4(_ptr(packed), _ptr(_c(s_bits, np.uint16)), _ptr(_c(z_bits, np.uint16)),
                                    N, K, _ptr(out))
        return out

    def ec_gate(self, x_bits, A_bits, wg_bits, b_g: float):
        """t = x A, p = x w_g + b_g, g = sigmoid(p) (fp64).  Returns (t [M,r], p [M], g [M])."""
        x_bits = _c(x_bits, np.uint16)
        A_bits = _c(A_bits, np.uint16)
        M, K = x_bits.shape
        r = A_bits.shape[1]
        t = np.empty((M, r), np.float64)
        p = np.empty(M, np.float64)
        g = np.empty(M, np.float64)
        self._lib.oracle_ec_gate(_ptr(x_bits), M, K, _ptr(A_bits), r, _ptr(_c(wg_bits, np.uint16)),
                                 ctypes.c_float(b_g), _ptr(t), _ptr(p), _ptr(g))
        return t, p, g

    def w4ec_gemm(self, x_bits, packed, s_bits, z_bits, A_bits=None, B_bits=None, wg_bits=None,
                  b_g: float = 0.0) -> np.ndarray:
        """The whole layer in fp64: y [M,N].  A_bits None -> plain W4 layer."""
        x_bits = _c(x_bits, np.uint16)
        packed = _c(packed, np.uint8)
        M, K = x_bits.shape
        N = packed.shape[0]
        r = 0 if A_bits is None else int(np.shape(A_bits)[1])
        y = np.empty((M, N), np.float64)
        self._lib.oracle_w4ec_gemm(_ptr(x_bits), M, N, K, _ptr(packed), _ptr(_c(s_bits, np.uint16)),
                                   _ptr(_c(z_bits, np.uint16)), _ptr(_c(A_bits, np.uint16)),
                                   _ptr(_c(B_bits, np.uint16)), _ptr(_c(wg_bits, np.uint16)),
                                   ctypes.c_float(b_g), r, _ptr(y))
        return y

    def pack_w4_grouped(self, W: np.ndarray, G: int):
        """Group-wise RTN: the per-channel format of W viewed as [N * K/G, G].
        Returns packed [N, K/2], s and z binary16 bits [N, K/G]."""
        N, K = W.shape
        packed, s, z = self.pack_w4(np.ascontiguousarray(W, dtype=np.float32).reshape(N * (K // G), G))
        return packed.reshape(N, K // 2), s.reshape(N, K // G), z.reshape(N, K // G)

    def w4ec_gemm_grouped(self, x_bits, packed, s_bits, z_bits, G: int, A_bits=None, B_bits=None, wg_bits=None,
                          b_g: float = 0.0):
        """y fp64 [M, N] of the layer with group-wise scales (s, z [N, K/G]); no EC if A_bits is None."""
        x = _c(x_bits, np.uint16)
        M, K = x.shape
        N = packed.shape[0]
        r = 0 if A_bits is None else A_bits.shape[1]
        y = np.empty((M, N), dtype=np.float64)
        self._lib.oracle_w4ec_gemm_grouped(
            _ptr(x), M, N, K, G, _ptr(_c(packed, np.uint8)), _ptr(_c(s_bits, np.uint16)), _ptr(_c(z_bits, np.uint16)),
            None if A_bits is None else _ptr(_c(A_bits, np.uint16)),
            None if B_bits is None else _ptr(_c(B_bits, np.uint16)),
            None if wg_bits is None else _ptr(_c(wg_bits, np.uint16)), b_g, r, _ptr(y))
        return y

    def w4ec_gemm_mlp(self, x_bits, packed, s_bits, z_bits, A_bits, B_bits, W1, b1, W2, b2, alpha: float = 1.0):
        """The layer with the bottleneck-MLP gate (see oracle_w4ec_gemm_mlp): fp64 y [M, N]."""
        x_bits = _c(x_bits, np.uint16)
        M, K = x_bits.shape
        N = packed.shape[0]
        A_bits, B_bits = _c(A_bits, np.uint16), _c(B_bits, np.uint16)
        r = A_bits.shape[1]
        W1, b1, W2, b2 = (_c(a, np.float32) for a in (W1, b1, W2, b2))
        H = W1.shape[0]
        assert W1.shape == (H, r) and b1.shape == (H,) and W2.shape == (r, H) and b2.shape == (r,)
        y = np.empty((M, N), dtype=np.float64)
        self._lib.oracle_w4ec_gemm_mlp(_ptr(x_bits), M, N, K, _ptr(_c(packed, np.uint8)), _ptr(_c(s_bits, np.uint16)),
                                      _ptr(_c(z_bits, np.uint16)), _ptr(A_bits), _ptr(B_bits), r, _ptr(W1), _ptr(b1),
                                      _ptr(W2), _ptr(b2), H, ctypes.c_float(alpha), _ptr(y))
        return y

    def w4ec_gemm_sampled(self, x_bits, packed, s_bits, z_bits, A_bits, B_bits, wg_bits, b_g,
                          mi, ni) -> np.ndarray:
        """The layer evaluated at the sampled outputs (mi[c], ni[c]) only."""
        x_bits = _c(x_bits, np.uint16)
        packed = _c(packed, np.uint8)
        M, K = x_bits.shape
        N = packed.shape[0]
        r = 0 if A_bits is None else int(np.shape(A_bits)[1])
        mi = _c(mi, np.int64)
        ni = _c(ni, np.int64)
        y = np.empty(len(mi), np.float64)
        self._lib.oracle_w4ec_gemm_sampled(_ptr(x_bits), M, N, K, _ptr(packed), _ptr(_c(s_bits, np.uint16)),
                                           _ptr(_c(z_bits, np.uint16)), _ptr(_c(A_bits, np.uint16)),
                                           _ptr(_c(B_bits, np.uint16)), _ptr(_c(wg_bits, np.uint16)),
                                           ctypes.c_float(b_g), r, _ptr(mi), _ptr(ni), len(mi), _ptr(y))
        return y


def default() -> Oracle:
    """The oracle built from ``spear_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def __getattr__(name):
    # Module-level shortcuts: oracle.pack_w4(...) etc. call the default build.
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)
