"""CPU oracle (float64) for the absorbed sparse-MLA decode path.

Test infrastructure: imported only by the tests, the smoke check and the
bench's CPU-baseline leg; never by the CUDA library or its Python binding.
"""
from .mla_oracle import (  # noqa: F401
    apply_wuv,
    cache_write,
    decode_absorbed,
    decode_materialised,
    decode_multi_query,
    expand_keys_values,
    fold_wuk,
    index_mask,
    mix_latent,
    out_proj,
    parameter_counts,
    prefill_mask,
    prefill_materialised,
    query_proj,
    rmsnorm,
    rope,
    scores,
    selected_positions,
    softmax_rows,
)
