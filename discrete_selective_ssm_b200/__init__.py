"""B200-native (sm_100a) Naju scan: conv + SiLU, selective scan, readout,
SiLU(z) modulation, backward and decode step, as a C-ABI CUDA library with a
thin Python binding.

The binding loads ``libnaju.so`` (built in-tree by
``discrete_selective_ssm_b200.build``) on first use and raises if it cannot;
there is no fallback path.  ``workloads`` (seeded synthetic inputs) imports
nothing from the binding.
"""
from ._native import (BF16, F32, Dims, NajuError, alloc_workspace, conv_silu_bwd,  # noqa: F401
                      conv_silu_fwd, conv_silu_step, declared_symbols, last_device_status, lib,
                      library_path, make_dims, scan_bwd, scan_fwd, scan_step, scan_step_conv,
                      testing_bwd_groups, testing_bwd_impl, testing_bwd_pieces,
                      testing_fwd_groups, testing_fwd_impl, testing_fwd_pieces,
                      testing_set_bwd_groups, testing_set_bwd_impl, testing_set_bwd_pieces,
                      testing_set_fwd_groups, testing_set_fwd_impl, testing_set_fwd_pieces,
                      testing_set_skip_publish, testing_set_sm_count, testing_set_wait_limit,
                      testing_sm_count, workspace_bytes)
