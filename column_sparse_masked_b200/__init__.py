"""Column-sparse masked attention (FlashMask encoding) for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libflashmask.so`` (declared in
``include/flashmask.h``): argument marshalling only.  Every step of the
computation runs in the library's CUDA kernels; PyTorch provides device
memory (outputs and workspace) and the current stream.  There is no CPU or
PyTorch fallback: if the library cannot be loaded, every call raises.

Method: "FlashMask-3 targets masked distributed attention on Hopper GPUs",
section "In-depth insight" -- a structured mask stored column-wise as four
query-axis boundary vectors per key column (LTS, LTE, UTS, UTE); row i is
masked for key j iff LTS[j] <= i < LTE[j] or UTS[j] <= i < UTE[j].

Layouts: q/o/dO/dq ``[B, Nq, Hq, d]``, k/v/dk/dv ``[B, Nk, Hkv, d]`` (bf16,
contiguous), lse ``[B, Hq, Nq]`` fp32, mask vectors ``[B, Hm, Nk]`` int32 with
Hm in {1, Hq}.  A ``None`` pair (lts/lte or uts/ute) means empty intervals.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    FlashMaskError,
    balance_chunks,
    classify,
    count_unmasked,
    flashmask_attention,
    fwd,
    bwd,
    get_status,
    get_timeout_info,
    launch_count,
    lib_path,
    load_library,
    localize,
    localize_multi,
    merge_partials,
    profiler_enable,
    profiler_read,
    get_bwd_mode,
    get_fwd_pairing,
    set_bwd_mode,
    set_fwd_pairing,
    set_max_ctas,
    set_wait_limit_ns,
    test_wait_timeout,
    tile_costs,
    version,
    workspace_size,
)

__all__ = [
    "FlashMaskError", "balance_chunks", "classify", "count_unmasked", "flashmask_attention", "fwd", "bwd", "get_status", "get_timeout_info",
    "launch_count", "lib_path", "load_library", "localize", "localize_multi", "merge_partials", "profiler_enable", "profiler_read", "get_bwd_mode", "set_bwd_mode", "get_fwd_pairing", "set_fwd_pairing", "set_max_ctas", "set_wait_limit_ns", "test_wait_timeout", "tile_costs",
    "version", "workspace_size",
]
