"""Static SVD-initialised error compensator: an offline initialiser for the EC factors.

SPEAR technical summary, section 1: the compensators that precede SPEAR are static low-rank
corrections, the same for every token.  Their data-free form is the best rank-r approximation of
the weight error seen from the input side, (W - W_hat)^T ~= A B, with A = U_r diag(sqrt(s_r)) and
B = diag(sqrt(s_r)) V_r^T from its singular value decomposition, and the gate held at 1.  The layer
then computes y = x W_hat^T + x A B with the same kernels as the gated compensator.

This is calibration, not the layer's hot path: W_hat comes from the library's own unpacking of
the packed codes (``spear_debug_unpack_w4``, times the fp16 scales), and the decomposition is
PyTorch's (cuSOLVER) on the device.
"""
from __future__ import annotations

import torch

from . import EC, spear_debug_unpack_w4


def weight_error_t(W: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor) -> torch.Tensor:
    """(W - W_hat)^T in fp32, [K, N], on W's device.  (q - z) s is exact in fp32."""
    K = W.shape[1]
    _, qz = spear_debug_unpack_w4(packed, zero, K, want_q=False)
    W_hat = qz.float() * scale.float()[:, None]
    return (W.float() - W_hat).t().contiguous()


def svd_compensator(W: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor,
                    rank: int) -> EC:
    """The rank-`rank` static compensator of one layer as an EC (bf16 A [K, r], B [r, N]) whose
    gate is 1 for every token (w_g = 0, b_g = +inf)."""
    E_t = weight_error_t(W, packed, scale, zero)
    U, s, Vh = torch.linalg.svd(E_t.double(), full_matrices=False)
    root = s[:rank].sqrt()
    A = (U[:, :rank] * root).to(torch.bfloat16).contiguous()
    B = (root[:, None] * Vh[:rank]).to(torch.bfloat16).contiguous()
    w_g = torch.zeros(W.shape[1], dtype=torch.bfloat16, device=W.device)
    return EC(A, B, w_g, float("inf"))
