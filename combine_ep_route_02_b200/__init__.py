"""B200 (sm_100a) MoE expert-parallel routing, dispatch layout, FP8 dispatch
and weighted combine on one GPU.

The compute lives in ``lib/libep_b200.so`` (C ABI in ``include/ep.h``); this
package is its ctypes binding plus ``EpPath``, which owns the device buffers
for one shape.  Importing the package does not load the library; the first
call does, and raises if it has not been built.
"""

from ._binding import (  # noqa: F401
    EP_DEV_BAD_EXPERT,
    EP_DEV_BAD_REPLICA,
    EP_DEV_OVERFLOW,
    EP_DEV_TIMEOUT,
    EP_ERR_CUDA,
    EP_ERR_DEVICE,
    EP_ERR_INVALID,
    EP_ERR_UNSUPPORTED,
    EP_OK,
    EXPORTS,
    EpError,
    RouteCfg,
    ep_combine,
    ep_combine_backward,
    ep_dispatch_backward,
    ep_dispatch,
    ep_dispatch_layout,
    ep_route,
    ep_route_dispatch,
    ep_route_layout,
    ep_testing_set_wait_limit,
    ep_silu_mul,
    ep_workspace_size,
    lib,
)
from .exchange import (ExchangePlan, combine_exchange, dispatch_exchange,  # noqa: F401
                       exchange_plan)
from .path import EpHostPipeline, EpMicroBatchPipeline, EpPath  # noqa: F401
from .peer import EpPeerRanks  # noqa: F401
