"""B200 (sm_100a) absorbed sparse-MLA decode: Python binding of libshla.

The compute path is the CUDA library ``libshla.so`` built in-tree by
``sparse_head_latent_absorbed_b200.build``; this package only marshals
arguments (see ``_lib``).  There is no CPU fallback: the library is loaded
on first use of any name below, and that raises ImportError when it is not
built.  Importing the package itself (or its ``build`` module) does not need
the library, so a clean tree can build it.
"""
_EXPORTS = (
    "LIB",
    "LIB_PATH",
    "MLAError",
    "mla_cache_write",
    "mla_cache_write_noalloc",
    "mla_cache_write_workspace_bytes",
    "mla_decode",
    "mla_decode_mq",
    "mla_decode_num_splits",
    "mla_decode_phase",
    "mla_decode_workspace_bytes",
    "mla_fold_wuk",
    "mla_gather_rows",
    "mla_index_mask",
    "mla_out_proj",
    "mla_out_proj_workspace_bytes",
    "mla_query_proj",
    "mla_query_proj_workspace_bytes",
    "mla_rope",
    "mla_wait_limit_check",
    "status_string",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(list(globals()) + list(_EXPORTS))
