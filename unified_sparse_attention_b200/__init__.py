"""unified_sparse_attention_b200 -- LServe-style unified block-sparse attention on B200.

A thin Python binding over the C ABI of ``liblserve.so`` (``include/lserve.h``).
The functions here have the C entry points' names and do argument marshalling
only (dtype/shape/device checks, pointer extraction, workspace allocation through
PyTorch); every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: importing works without a GPU, but every call needs
the compiled library and a CUDA device, and raises otherwise.
"""
from .binding import (  # noqa: F401
    LServeError,
    LSERVE_HEAD_DENSE,
    LSERVE_HEAD_STREAMING,
    library_path,
    load_library,
    lserve_decode,
    lserve_decode_max_selected,
    lserve_decode_noalloc,
    lserve_decode_reuse,
    lserve_decode_int4,
    lserve_quantize_pages_int4,
    lserve_cra,
    lserve_cra_workspace_size,
    lserve_build_vslash_mask,
    lserve_vslash_workspace_size,
    lserve_decode_workspace_size,
    lserve_get_device_status,
    lserve_last_error_string,
    lserve_prefill,
    lserve_prefill_tile_lists,
    lserve_prefill_workspace_size,
    lserve_update_page_stats,
    lserve_version,
    EXPORTED_SYMBOLS,
)
