"""B200-native hot path of one joint video + audio DiT block: fused Q/K
RMSNorm + RoPE, packed variable-length attention on tcgen05 tensor cores,
and fused adaLN modulation + gated residual + SwiGLU, behind the C ABI in
include/pqk.h (libpqk.so, built by ``packed_attention_qk_b200.build``)."""

from .pqk import (  # noqa: F401
    NORM_LAYER, NORM_NONE, NORM_RMS, ROPE_HALF, ROPE_INTERLEAVED, PqkError, get_device_status, modulate_swiglu,
    qk_fullc_norm_rope, qk_norm_rope, qk_norm_rope_3axis, selftest_wait_timeout, set_wait_timeout_ns, varlen_attn_fwd, varlen_attn_workspace_size, version,
)
