"""B200-native (sm_100a) on-device MoE expert-parallel dispatch and combine.

The kernels live in ``libmoe.so`` behind the C ABI of ``include/moe.h``; this
package is a thin ctypes binding with the same names (``route_topk``,
``demand_hist``, ``replica_assign``, ``build_layout``, ``pack``, ``combine``)
plus ``DispatchCombine``, which runs the whole path with preallocated buffers,
and ``HostPipeline``, which runs it on pinned host inputs and outputs with the
copies overlapped with the kernels.
There is no CPU fallback: calls raise if the library is not built.
"""
from ._binding import (BF16, DEDUP, F16, F32, MOE_OK, PER_PICK, STATUS_NAMES, TWO_HOP, LIB_PATH,  # noqa: F401
                       Layout, MoeError, build_layout, check_status, combine, debug_set_wait,
                       demand_hist, get_status, kernel_launches, layout_workspace_size, lib, moe_layout, pack,
                       replica_assign, route_topk, status_string, dispatch_stats,
                       token_balanced_assign, STAT_NAMES, route_layout_single_replica, route_assign_layout,
                       coselection_hist, correlated_placement)
from .path import DispatchCombine, HostPipeline  # noqa: F401
