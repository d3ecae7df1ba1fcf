"""B200 (sm_100a) fused mixture-of-experts expert forward.

The compute lives in libmoe_b200.so (C ABI: include/moe.h); this package is a
thin ctypes binding over it plus seeded synthetic workloads.  Importing the
package does not load the library; the first call does, and raises if the
library was not built (there is no CPU fallback).
"""

from ._abi import (MoeConfig, MoeError, MoeTensor, MoeW13, align, builtin_config_count,  # noqa: F401
                   config_override, desc, device_errors, forward, forward_host, forward_status,
                   get_config, last_launch_count, load, make_config, profile_enable, profile_read,
                   quantize_mxfp4, router_status, router_topk, set_config_table, version, w13_from_packed, w13_from_views,
                   workspace_bytes, workspace_layout, debug_capture, MOE_CAPTURE_H_PREQUANT,
                   measure_mma_peak, backward, backward_input, backward_status, backward_workspace_bytes,
                   transpose_experts, host_workspace_bytes)
