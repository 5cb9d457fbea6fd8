"""fp64 oracle of the token-phase attention step -- TEST INFRASTRUCTURE ONLY.

Source: "FastTPS: An Optimized Method for LLM Token Phase for AI
Accelerators" (xllm-io paper review), section 三 "技术架构", components 1-2
and Figure 3: GKVC keeps one preallocated KV-cache region per head and
writes the new token's K and V straight into it at the address given by
Eq(2), so no Concat ever rebuilds the cache; TPSFLAT computes the
attention of the new token over the cache in tiles, with RoPE, Q K^T,
Softmax and P V fused.

Restated plainly (readings where the pages are silent are marked *):

  * cache layout: head-major, one region of N_max = N_p + N_r rows of d
    values per KV head; Eq(2) gives the element offset of the new row as
    Step = h (N_p + N_r) d + N_p d, with N_p the rows already held (the new
    token's position) and N_p + N_r the region's capacity.  Sequences of a
    batch follow one another (*).
  * RoPE (*: the "rotate-half" pairing, element i with element i + d/2, and a
    base theta): angle_i = pos * theta^(-2i/d), i < d/2,
        x'[i]       = x[i] cos(angle_i) - x[i + d/2] sin(angle_i)
        x'[i + d/2] = x[i] sin(angle_i) + x[i + d/2] cos(angle_i).
    Applied to the new token's q and k at its position.
  * the stored K row is the rotated k rounded to bf16 (*: the cache holds
    bf16, like the weights), the stored V row is v itself;
  * attention of each query head h over rows 0..pos (the new row included),
    with KV head g = h // (H / H_kv) (*: grouped queries share a KV head):
        s_j = scale * q'_h . K_g[j],  p = softmax(s),  o_h = sum_j p_j V_g[j]
    and scale = 1/sqrt(d) (*).
"""

from __future__ import annotations

import numpy as np

from .fmlp import round_to_bf16


def gkvc_step(h: int, n_p: int, n_r: int, d: int) -> int:
    """Eq(2): element offset of the new row of KV head h in a region of
    n_p + n_r rows of d values per head, n_p rows already written."""
    return h * (n_p + n_r) * d + n_p * d


def rope_angles(pos: int, d: int, theta: float) -> np.ndarray:
    """angle_i = pos * theta^(-2i/d) for i < d/2 (binary64)."""
    if d % 2:
        raise ValueError("RoPE needs an even head dimension")
    i = np.arange(d // 2, dtype=np.float64)
    return float(pos) * np.power(float(theta), -2.0 * i / d)


def rope(x, pos: int, theta: float) -> np.ndarray:
    """Rotate each pair (x[i], x[i + d/2]) of the last axis by angle_i."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    a = rope_angles(pos, d, theta)
    c, s = np.cos(a), np.sin(a)
    lo, hi = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([lo * c - hi * s, lo * s + hi * c], axis=-1)


def decode_attention(q_rot, K, V, scale: float) -> np.ndarray:
    """o [H, d] for rotated queries q_rot [H, d] over K, V [H_kv, n, d]."""
    q_rot = np.asarray(q_rot, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    H, d = q_rot.shape
    H_kv = K.shape[0]
    if H % H_kv:
        raise ValueError("query heads must be a multiple of KV heads")
    group = H // H_kv
    out = np.empty((H, d))
    for h in range(H):
        g = h // group
        s = scale * (K[g] @ q_rot[h])
        w = np.exp(s - np.max(s))
        w /= np.sum(w)
        out[h] = w @ V[g]
    return out


def kv_append(cache, row, pos: int) -> np.ndarray:
    """A copy of cache [H_kv, N_max, d] with row [H_kv, d] written at
    position pos of every head, addressed by Eq(2) on the flat region."""
    cache = np.array(cache, dtype=np.float64)
    H_kv, n_max, d = cache.shape
    if not 0 <= pos < n_max:
        raise ValueError("position outside the cache region")
    flat = cache.reshape(-1)
    for h in range(H_kv):
        o = gkvc_step(h, pos, n_max - pos, d)
        flat[o:o + d] = row[h]
    return flat.reshape(H_kv, n_max, d)


def token_attention(q, k_new, v_new, k_cache, v_cache, pos, theta: float,
                    scale: float | None = None):
    """One token-phase attention step for a batch of B sequences.

    q [B, H, d], k_new / v_new [B, H_kv, d] (values of the new token, before
    RoPE), k_cache / v_cache [B, H_kv, N_max, d], pos [B] (rows already held).
    Returns (o [B, H, d], k_cache', v_cache') with the new rows appended."""
    q = np.asarray(q, dtype=np.float64)
    B, H, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    ko = np.empty(np.shape(k_cache))
    vo = np.empty(np.shape(v_cache))
    out = np.empty((B, H, d))
    for b in range(B):
        p = int(pos[b])
        k_row = round_to_bf16(rope(k_new[b], p, theta))
        ko[b] = kv_append(k_cache[b], k_row, p)
        vo[b] = kv_append(v_cache[b], np.asarray(v_new[b], dtype=np.float64), p)
        out[b] = decode_attention(rope(q[b], p, theta), ko[b][:, : p + 1],
                                  vo[b][:, : p + 1], scale)
    return out, ko, vo
