"""B200 (sm_100a) forward and backward passes of 1D deformable convolution (DeformConv1d)
and PackedDeformConv1d's forward (offsets and mask predicted inside the layer).

The computation lives in the C-ABI CUDA library ``libdcn1d.so`` (declared in
``include/dcn1d.h``); this package is its thin Python binding.
"""
from ._binding import (  # noqa: F401
    DCN1D_BF16,
    DCN1D_F16,
    DCN1D_F32,
    Dcn1dError,
    Dcn1dTensor,
    GRADS,
    SIGNATURES,
    clear_workspace_cache,
    dcn1d_backward,
    dcn1d_backward_kernel_name,
    dcn1d_backward_workspace_size,
    dcn1d_device_status,
    dcn1d_forward,
    dcn1d_forward_noalloc,
    dcn1d_forward_workspace_size,
    dcn1d_forward_kernel_name,
    dcn1d_last_launch_count,
    dcn1d_out_length,
    dcn1d_packed_forward,
    dcn1d_packed_forward_kernel_name,
    dcn1d_packed_trunk,
    dcn1d_packed_trunk_kernel_name,
    dcn1d_sample_index,
    dcn1d_set_timing_events,
    dcn1d_status_string,
    lib_path,
    load,
    resolve_padding,
)
