"""AnchorKV anchor-residual KV-cache codec for NVIDIA B200 (sm_100a).

The codec runs in the CUDA library libanchorkv.so (C ABI: include/anchorkv.h);
this package is its PyTorch binding.  Importing the package does not load the
library; the first call does, and fails loudly if it has not been built.
"""
from .api import (AnchorKVParams, HostCompressor, anchorkv_bytes, codebook, compress, compress_host,
                  compress_host_staging_bytes, compress_workspace,
                  decode_attn, decode_workspace_bytes, read_status, reconstruct)

__all__ = ["AnchorKVParams", "HostCompressor", "anchorkv_bytes", "codebook", "compress", "compress_host",
           "compress_host_staging_bytes", "compress_workspace",
           "decode_attn", "decode_workspace_bytes", "read_status", "reconstruct"]
