"""fp64 oracle of the int8 weight format -- TEST INFRASTRUCTURE ONLY.

The pages name quantized weight streaming over interleaved gate/up rows (the
llama.cpp PR #29948 paragraph of "CUDAカーネル融合で推論が最大10%高速化",
blog.cecily.jp: MMQ with the fused gate/up + GLU, Q4_K_M) but define no
block format.  The library's own format, restated here plainly:

  * a weight matrix W [rows x K] (K: the contraction axis -- d for the packed
    gate/up rows, I for W_down) is cut along K into groups of G = 64
    consecutive elements of one row;
  * each group g has one binary32 scale  s_g = fl32(max_k |w_k| / 127)
    (IEEE binary32 division, round to nearest even); s_g = 0 for a group of
    zeros;
  * each weight is the int8  q_k = clamp(rint(fl32(w_k / s_g)), -127, 127),
    the division in binary32 and rint rounding halves to even (q_k = 0 when
    s_g = 0);
  * the weight it stands for is q_k * s_g, exactly.

Quantization is row-wise, so it commutes with the gate/up row interleave:
quantizing the packed matrix equals packing the quantized matrices.  The block
computed on quantized weights is the block of Eq(1) (see ``fmlp.py``) on the
dequantized weights.
"""

from __future__ import annotations

import numpy as np

from .fmlp import fused_mlp

GROUP = 64


def quantize_rows(W, group: int = GROUP):
    """(q int8 [rows x K], s float32 [rows x K/group]) of W [rows x K] (values
    exactly representable in binary32, e.g. decoded bf16)."""
    W = np.asarray(W, dtype=np.float64)
    rows, K = W.shape
    if K % group != 0:
        raise ValueError(f"K = {K} is not a multiple of the group size {group}")
    w32 = W.astype(np.float32)
    if not np.array_equal(w32.astype(np.float64), W):
        raise ValueError("weights must be exactly representable in binary32")
    g = w32.reshape(rows, K // group, group)
    m = np.max(np.abs(g), axis=2)                           # exact
    s = (m / np.float32(127.0)).astype(np.float32)          # binary32 division, RN
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (g / s[:, :, None]).astype(np.float32)          # binary32 division, RN
    q = np.where(s[:, :, None] > 0, np.clip(np.rint(r), -127, 127), 0.0)
    return q.reshape(rows, K).astype(np.int8), s


def dequantize_rows(q, s, group: int = GROUP) -> np.ndarray:
    """q * s in binary64 (exact: an int8 times a binary32)."""
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    rows, K = q.shape
    return (q.reshape(rows, K // group, group) * s[:, :, None]).reshape(rows, K)


def fused_mlp_q8(x, gamma, eps, Wg_q, Wg_s, Wu_q, Wu_s, Wd_q, Wd_s, residual=None,
                 intermediate=None, group: int = GROUP) -> np.ndarray:
    """The MLP block on int8 weights: Eq(1) with RMSNorm on the dequantized
    W_gate, W_up [I x d] and W_down [d x I]."""
    return fused_mlp(x, gamma, eps, dequantize_rows(Wg_q, Wg_s, group),
                     dequantize_rows(Wu_q, Wu_s, group), dequantize_rows(Wd_q, Wd_s, group),
                     residual=residual, intermediate=intermediate)
