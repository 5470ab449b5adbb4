"""Chunkwise Gated DeltaNet (gated delta rule) forward and backward for NVIDIA B200.

The computation runs in hand-written sm_100a CUDA kernels behind the C ABI in
include/gdn.h (libgdn_b200.so); this package is the thin Python binding.
"""
from .binding import (GDNError, gdn_build_chunk_indices, gdn_chunk_bwd, gdn_chunk_fwd,
                      gdn_chunk_table_device, gdn_device_status, gdn_dims, gdn_recurrent_fwd,
                      gdn_kda_recurrent_fwd, gdn_kda_chunk_fwd, gdn_kda_chunk_bwd,
                      kda_chunk_workspace_bytes, state_affine,
                      kda_gate_bwd, kda_gate_fwd, kda_gate_workspace_bytes,
                      make_dims, max_chunks, recurrent_workspace_bytes, status_string, version,
                      workspace_bytes, launch_count, profile, profile_read)

__all__ = ["GDNError", "gdn_build_chunk_indices", "gdn_chunk_bwd", "gdn_chunk_fwd",
           "gdn_chunk_table_device", "gdn_device_status", "gdn_dims", "make_dims", "max_chunks",
           "status_string", "version", "workspace_bytes", "launch_count", "profile",
           "profile_read", "gdn_recurrent_fwd", "recurrent_workspace_bytes", "kda_gate_fwd",
           "kda_gate_bwd", "kda_gate_workspace_bytes", "gdn_kda_recurrent_fwd", "gdn_kda_chunk_fwd", "gdn_kda_chunk_bwd",
           "kda_chunk_workspace_bytes", "state_affine"]
