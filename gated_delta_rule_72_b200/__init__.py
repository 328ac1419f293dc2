"""B200-native (sm_100a) gated delta-net scan: causal, bidirectional, streaming step.

The compute path is libgdn.so (hand-written CUDA kernels behind a C-ABI,
include/gdn.h).  This package binds it with ctypes (`_lib`, same names as
the C functions) and adds torch-facing wrappers (`api`).  There is no CPU
fallback: calls fail loudly if the library is not built or the tensors are
not on a CUDA device.
"""
from ._lib import GDNError, gdn_scan_bidir, gdn_scan_bidir_states, gdn_scan_causal, gdn_status_string, gdn_step, \
    gdn_version, gdn_workspace_size, gdn_launch_count, gdn_set_kernel_timing, \
    gdn_read_kernel_timing, gdn_device_timeouts, gdn_set_short_call_tokens, gdn_set_chain_segments, gdn_readout_gate, gdn_vda_scan, gdn_vda_workspace_size, load  # noqa: F401
from .api import readout_gate, scan_bidir, scan_causal, step, vda_scan, workspace_size  # noqa: F401
