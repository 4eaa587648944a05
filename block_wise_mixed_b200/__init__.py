"""block_wise_mixed_b200 -- block-wise mixed-precision weight-only quantized
linear layer (64x128 blocks, per-block bits in {0,1,2,3,4,5,6,8} plus 16-bit passthrough blocks, RTN-g128,
fp16 scale/zero, bi-directional channel reordering) on NVIDIA B200.

The computation lives in the C-ABI library ``libmpq.so`` (include/mpq.h); this
package only marshals arguments to it.  ``synth`` draws seeded workloads.
"""
from ._lib import (GROUP_MAX, Y_BF16, Y_F32, MpqError, PackedLayer, allocate_bits, check, fold_orders,  # noqa: F401
                   linear,
                   linear_group, linear_group_workspace_size, linear_host, linear_host_workspace_size,
                   linear_timed, linear_typed_workspace_size, linear_workspace_size, pack, plan,
                   with_orders)
