"""B200 (sm_100a) absorbed sparse-MLA decode: Python binding of libshla.

The compute path is the CUDA library ``libshla.so`` built in-tree by
``sparse_head_latent_absorbed_b200.build``; this package only marshals
arguments (see ``_lib``).  There is no CPU fallback: importing the package
without the built library raises ImportError.
"""
from ._lib import (  # noqa: F401
    LIB,
    LIB_PATH,
    MLAError,
    mla_cache_write,
    mla_cache_write_noalloc,
    mla_cache_write_workspace_bytes,
    mla_decode,
    mla_decode_mq,
    mla_decode_num_splits,
    mla_decode_phase,
    mla_decode_workspace_bytes,
    mla_fold_wuk,
    mla_gather_rows,
    mla_index_mask,
    mla_out_proj,
    mla_out_proj_workspace_bytes,
    mla_query_proj,
    mla_query_proj_workspace_bytes,
    mla_rope,
    status_string,
)
