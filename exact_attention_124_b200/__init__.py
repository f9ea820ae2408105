"""B200-native exact attention forward.

The work happens in ``libattn_b200.so`` (hand-written sm_100a CUDA behind the
C ABI in ``include/attn.h``); this package only marshals torch tensors
(device memory and streams) into that ABI.  There is no fallback: if the
library is missing every call raises.
"""
from ._lib import (AttnError, bwd, decode_plan, fused_plan, fwd, fwd_decode, fwd_gqa, fwd_host, fwd_unfused, last_error, library_path,
                   load_library, selftest_pv_tile, selftest_qk_tile, selftest_timeout,
                   set_exp_split, set_mma_order, status_str, fused_grid_ctas, unfused_workspace_bytes, version)
from .autograd import attention

__all__ = ["AttnError", "attention", "bwd", "decode_plan", "fused_plan", "fwd", "fwd_decode", "fwd_gqa", "fwd_host", "fwd_unfused", "last_error", "library_path",
           "load_library", "selftest_pv_tile", "selftest_qk_tile", "selftest_timeout",
           "set_exp_split", "set_mma_order", "status_str", "fused_grid_ctas", "unfused_workspace_bytes", "version"]
