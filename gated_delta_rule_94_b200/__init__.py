"""Gated delta-rule linear attention on NVIDIA B200 (sm_100a).

The operator runs in libgdn.so (C ABI in include/gdn.h); this package holds
its thin ctypes binding (:mod:`._lib`), the in-tree build script
(:mod:`.build`) and the seeded synthetic-input generator (:mod:`.inputs`).
"""
from ._lib import (GDN_BF16, GDN_F32, GDN_GATE_NONE, GDN_GATE_PER_DIM, GDN_GATE_SCALAR,  # noqa: F401
                   GdnError, chunk_fwd, decode_step, gdn_abi_version, gdn_chunk_fwd,
                   gdn_chunk_fwd_wk, gdn_osdn_precondition, gdn_osdn_precondition_workspace_bytes,
                   osdn_chunk_fwd, gdn_chunk_fwd_plan,
                   chunk_bwd, gdn_chunk_bwd, gdn_chunk_bwd_workspace_bytes,
                   gdn_chunk_fwd_workspace_bytes, gdn_chunk_fwd_workspace_min_bytes,
                   gdn_decode_step,
                   gdn_kernel_launch_count, gdn_chunk_fwd_kernel_name, gdn_read_device_status,
                   gdn_status_string)
