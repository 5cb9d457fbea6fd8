"""fp64 oracle of RMSNorm + Eq(1) + the gate/up row interleave.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain numpy in binary64;
matrix products use numpy's ``@`` as a library primitive and nothing is
blocked, fused or reordered beyond the definitions below.

Sources, cited by page title and section:
  [FastTPS]  "FastTPS: An Optimized Method for LLM Token Phase for AI
             Accelerators" (xllm-io paper review):
             section 三 技术架构 -- Eq(1), the MLP execution flow
             (RMSNorm -> interleaved gate-up Matmul -> siLu_Mul -> down
             projection), component 3 "Fusion MLP", Figure 4 parts 1-3;
             section 五 代码实现分析 -- Fusion MLP Steps 1-3;
             section 六 精度保证 -- bf16 simulation against a float baseline.
  [llama.cpp] "CUDAカーネル融合で推論が最大10%高速化、その効果と落とし穴"
             (blog.cecily.jp) -- the llama.cpp PR #29948 paragraph: gate and
             up rows placed alternately so one matmul pass yields both and the
             GLU is applied in the same pass.
"""

from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# bf16 <-> binary64
# ----------------------------------------------------------------------------

def decode_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> their exact values as float64.

    A bf16 number is the high 16 bits of an IEEE binary32 word, so the value is
    recovered exactly by placing the 16 bits on top of 16 zero bits.
    """
    b = np.ascontiguousarray(bits).view(np.uint16)
    with np.errstate(invalid="ignore"):     # signalling-nan patterns stay nan
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


_BF16_MAX = float.fromhex("0x1.fep127")   # largest finite bf16
_MIN_NORMAL = 2.0 ** -126                 # smallest normal binary32 / bf16


def round_to_bf16(v) -> np.ndarray:
    """float64 -> the nearest bf16 value (ties to even), returned as float64.

    bf16 keeps 8 significant bits and binary32's exponent range.  A finite
    value v = m * 2**e with 0.5 <= |m| < 1 rounds to rint(m * 2**8) * 2**(e-8);
    below the normal range the grid spacing is fixed at 2**-133.  Results past
    the largest finite bf16 (after rounding) become +-inf; nan stays nan.
    ``np.rint`` rounds halfway cases to even.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty_like(v)
    finite = np.isfinite(v)
    out[~finite] = v[~finite]
    f = v[finite]
    m, e = np.frexp(f)
    normal = np.abs(f) >= _MIN_NORMAL
    r = np.where(normal,
                 np.ldexp(np.rint(np.ldexp(m, 8)), e - 8),
                 np.ldexp(np.rint(np.ldexp(f, 133)), -133))
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[finite] = r
    return out


# ----------------------------------------------------------------------------
# The MLP block (Eq(1) with its RMSNorm prologue)
# ----------------------------------------------------------------------------

def rms_inv(x: np.ndarray, eps: float) -> np.ndarray:
    """Per-row reciprocal RMS: r[m] = 1 / sqrt(mean_k x[m,k]^2 + eps).

    [FastTPS] Fusion MLP Step 1 / Figure 4 part 1 name RMSNorm without a
    formula; this is the standard reading: mean over the hidden dimension,
    eps inside the square root.
    """
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """h = x * r * gamma with r from ``rms_inv`` (gamma multiplies directly)."""
    x = np.asarray(x, dtype=np.float64)
    return x * rms_inv(x, eps)[..., None] * np.asarray(gamma, dtype=np.float64)


def silu(t: np.ndarray) -> np.ndarray:
    """SiLU(t) = t / (1 + exp(-t)).

    For t very negative exp(-t) overflows to +inf and the quotient is -0, the
    IEEE limit; that overflow is expected and silenced.
    """
    t = np.asarray(t, dtype=np.float64)
    with np.errstate(over="ignore"):
        return t / (1.0 + np.exp(-t))


def swiglu_intermediate(h, W_gate, W_up) -> np.ndarray:
    """a = SiLU(h W_gate^T) * (h W_up^T) for token rows h [M x d] -> [M x I].

    [FastTPS] Eq(1) inner part and the siLu_Mul step: SiLU on the gate branch,
    elementwise product with the up branch.
    """
    h = np.asarray(h, dtype=np.float64)
    g = h @ np.asarray(W_gate, dtype=np.float64).T
    u = h @ np.asarray(W_up, dtype=np.float64).T
    return silu(g) * u


def gated_mlp(h, W_gate, W_up, W_down, intermediate=None) -> np.ndarray:
    """Eq(1) of [FastTPS] for token rows h [M x d]:  O = (SiLU(h Wg^T) * (h Wu^T)) Wd^T.

    SiLU acts on the gate branch and the product with the up branch is taken
    before the down projection (Eq(1); section 五 Step 3 lists the multiply
    next to W_down, Eq(1) fixes the order).  No bias terms.

    ``intermediate='bf16'`` rounds a = SiLU(g) * u to bf16 before the down
    projection -- the precision of the intermediate the fused design stores
    (the bf16 simulation of section 六).  The default keeps a in binary64.
    """
    a = swiglu_intermediate(h, W_gate, W_up)
    if intermediate == "bf16":
        a = round_to_bf16(a)
    elif intermediate is not None:
        raise ValueError(f"unknown intermediate precision {intermediate!r}")
    return a @ np.asarray(W_down, dtype=np.float64).T


def fused_mlp(x, gamma, eps, W_gate, W_up, W_down, residual=None,
              intermediate=None, output=None) -> np.ndarray:
    """The whole MLP block: RMSNorm -> Eq(1) -> optional residual add.

    [FastTPS] MLP execution flow: RMSNorm -> gate-up -> siLu_Mul -> down
    projection.  ``residual`` (same shape as the output) is added after the
    down projection when given.

    ``output='bf16'`` returns the block's result rounded once to bf16 (round
    to nearest, ties to even) after the residual add: the output that the
    next layer reads as its input when layers are chained in bf16 (the bf16
    simulation of [FastTPS] section 六 keeps tensors between operators in
    bf16).  The default returns the binary64 result.
    """
    h = rmsnorm(x, gamma, eps)
    O = gated_mlp(h, W_gate, W_up, W_down, intermediate=intermediate)
    if residual is not None:
        O = O + np.asarray(residual, dtype=np.float64)
    if output == "bf16":
        O = round_to_bf16(O)
    elif output is not None:
        raise ValueError(f"unknown output precision {output!r}")
    return O


# ----------------------------------------------------------------------------
# The gate/up interleave (a pure row permutation)
# ----------------------------------------------------------------------------

def interleaved_rows(I: int, T: int):
    """Packed-row positions of gate row i and up row i, for i in [0, I).

    [FastTPS] component 3 merges the gate and up projections into one matmul
    by interleaving their rows; [llama.cpp] places gate and up rows
    alternately (T = 1).  Tile granularity T generalises this: tile t holds
    gate rows tT..tT+w-1 followed by up rows tT..tT+w-1, with w = T except for
    a final partial tile of w = I mod T rows.
    """
    if T < 1:
        raise ValueError("tile T must be >= 1")
    i = np.arange(I, dtype=np.int64)
    t = i // T
    j = i - t * T
    w = np.minimum(T, I - t * T)
    base = 2 * T * t
    return base + j, base + w + j


def pack_gate_up(W_gate, W_up, T: int) -> np.ndarray:
    """P [2I x d]: P[gate_row(i)] = W_gate[i], P[up_row(i)] = W_up[i].

    Works on any dtype (bf16 bit patterns included): it only moves rows.
    """
    W_gate = np.asarray(W_gate)
    W_up = np.asarray(W_up)
    if W_gate.shape != W_up.shape or W_gate.ndim != 2:
        raise ValueError("W_gate and W_up must be equal-shape matrices")
    I, d = W_gate.shape
    gr, ur = interleaved_rows(I, T)
    P = np.empty((2 * I, d), dtype=W_gate.dtype)
    P[gr] = W_gate
    P[ur] = W_up
    return P


def unpack_gate_up(P, I: int, T: int):
    """Inverse of ``pack_gate_up``: (W_gate, W_up) read back through the permutation."""
    P = np.asarray(P)
    gr, ur = interleaved_rows(I, T)
    return P[gr], P[ur]


def fused_mlp_packed(x, gamma, eps, P, T, W_down, residual=None,
                     intermediate=None, output=None) -> np.ndarray:
    """The MLP block with gate/up weights read from the packed matrix P."""
    I = np.asarray(P).shape[0] // 2
    Wg, Wu = unpack_gate_up(P, I, T)
    return fused_mlp(x, gamma, eps, Wg, Wu, W_down, residual=residual,
                     intermediate=intermediate, output=output)


def fused_mlp_bf16(x_bits, gamma_bits, eps, Wg_bits, Wu_bits, Wd_bits,
                   residual_bits=None, intermediate=None, output=None) -> np.ndarray:
    """``fused_mlp`` fed bf16 bit patterns (the same bytes the GPU reads),
    each decoded exactly to binary64 first."""
    res = None if residual_bits is None else decode_bf16(residual_bits)
    return fused_mlp(decode_bf16(x_bits), decode_bf16(gamma_bits), float(eps),
                     decode_bf16(Wg_bits), decode_bf16(Wu_bits), decode_bf16(Wd_bits),
                     residual=res, intermediate=intermediate, output=output)
