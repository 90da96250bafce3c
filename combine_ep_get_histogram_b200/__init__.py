"""B200-native MoE expert-parallel dispatch / combine.

The hot path (routing layout, FP8/BF16 dispatch, combine and both backward
passes) runs in the CUDA library ``libep_b200.so`` behind the C ABI declared
in ``include/ep.h``; ``combine_ep_get_histogram_b200.ep`` is its thin ctypes
binding.  ``workloads`` draws the seeded synthetic inputs.
"""

from . import workloads  # noqa: F401  (inputs only; no method arithmetic)
from .ep import (  # noqa: F401
    EPError, Handle, make_shape, workspace, workspace_size, handle_sizes, library,
    ep_get_dispatch_layout, ep_get_dispatch_layout_noalloc, ep_dispatch, ep_dispatch_with_layout, ep_combine,
    ep_combine_backward, ep_dispatch_backward, ep_get_error, ep_route_group_limited, ep_dispatch_peers, ep_combine_peers,
    ep_combine_backward_peers, ep_dispatch_backward_peers, peer_rows,
)
