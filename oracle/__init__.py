"""fp64 CPU oracle for the fused gated MLP -- TEST INFRASTRUCTURE ONLY.

This package is the yardstick the CUDA library is checked against.  It is a
plain, slow, obviously correct restatement of the computation in binary64
numpy, written from the method's description and sharing no code, header,
table or helper with the CUDA path (``token_phase_swiglu_b200``), which it
never imports.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it;
the library itself must never route through it.

What it computes (sources: "FastTPS: An Optimized Method for LLM Token
Phase for AI Accelerators", xllm-io paper review, section 三 "技术架构":
Eq(1), the MLP-block execution flow and Figure 4; section 五 "Fusion MLP实现"
Steps 1-3; and "CUDAカーネル融合で推論が最大10%高速化" (blog.cecily.jp), the
llama.cpp PR #29948 paragraph on interleaved gate/up rows):

    r[m]   = 1 / sqrt(mean_k x[m,k]^2 + eps)                (RMSNorm, Step 1)
    h      = x * r * gamma
    g      = h W_gate^T,  u = h W_up^T                       (Eq(1) inner products)
    a      = SiLU(g) * u,  SiLU(t) = t / (1 + exp(-t))       (siLu_Mul)
    O      = a W_down^T  (+ residual, optional)              (down projection)

and the gate/up interleave, a pure permutation of rows at tile granularity.

``quant.py`` restates the library's own int8 weight format (the pages name
quantized weight streaming but give no format) and the block on it.

``attn.py`` restates the token-phase attention step of the same pages
(section 三, components 1-2 and Figure 3: GKVC's in-place KV append at the
Eq(2) address, TPSFLAT's RoPE + QK^T + Softmax + PV).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed
forms, exact invariants, brute force on tiny shapes and the page-described
row order -- never against the CUDA path.  No function here is "parity
unpinned".
"""

from .fmlp import (  # noqa: F401
    decode_bf16,
    round_to_bf16,
    rms_inv,
    rmsnorm,
    silu,
    swiglu_intermediate,
    gated_mlp,
    fused_mlp,
    interleaved_rows,
    pack_gate_up,
    unpack_gate_up,
    fused_mlp_packed,
    fused_mlp_bf16,
)
from .quant import (  # noqa: F401
    GROUP,
    quantize_rows,
    dequantize_rows,
    fused_mlp_q8,
)
from .attn import (  # noqa: F401
    gkvc_step,
    rope_angles,
    rope,
    decode_attention,
    kv_append,
    token_attention,
)
