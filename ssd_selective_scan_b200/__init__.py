"""B200-native (sm_100a) hot path of the Mamba-2 selective state-space layer.

libssd.so (built from csrc/ by ``python -m ssd_selective_scan_b200.build``)
holds the CUDA kernels behind the C ABI of include/ssd.h; ``binding`` is its
ctypes binding and ``layer`` the torch-facing calls.  The library is loaded
on first use and there is no fallback path: without libssd.so every call
raises.
"""
from .layer import (chunk_scan_bwd, chunk_scan_bwd_workspace_bytes, chunk_scan_fwd, chunk_scan_fwd_varlen, chunk_scan_varlen_workspace_bytes,
                    chunk_scan_workspace_bytes, conv1d_silu, conv_scan_fwd, conv_scan_workspace_bytes,
                    decode_step, layer_prefill, split_channels, state_update)
from .binding import SsdError

__all__ = ["chunk_scan_bwd", "chunk_scan_bwd_workspace_bytes", "chunk_scan_fwd", "chunk_scan_fwd_varlen", "chunk_scan_varlen_workspace_bytes",
           "chunk_scan_workspace_bytes", "conv1d_silu", "conv_scan_fwd", "conv_scan_workspace_bytes",
           "decode_step",
           "layer_prefill", "split_channels", "state_update", "SsdError"]
