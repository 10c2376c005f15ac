"""fp64 CPU oracle of the MLA decode step. Test infrastructure only (see mla_oracle)."""

from .mla_oracle import (  # noqa: F401
    cache_rows,
    rms_norm,
    D_HEAD,
    D_LATENT,
    D_ROPE,
    absorb_query,
    apply_wuv,
    default_scale,
    kv_cache_bytes,
    latent_attention,
    mha_cache_elements_per_token,
    mla_cache_elements_per_token,
    mla_decode_absorbed,
    mla_decode_nonabsorbed,
    rope_angles,
    rope_rotate,
    softmax_lse,
    token_rows,
    widen,
)
