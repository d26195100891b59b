"""B200-native (sm_100a) Kimi Delta Attention core.

Python binding of the C ABI in include/kda.h.  The entry points keep the
library's names:

  kda_chunk_fwd  chunk-parallel forward over whole sequences (o, S_T, M_T)
  kda_chunk_bwd  its gradient, from the per-chunk states the forward keeps
  kda_chunk      the two as a torch.autograd function (o, S_T)
  kda_step       single-token decode, state updated in place
  kda_compose    KCP segment prefix combine
  kcp_chunk_fwd  context-parallel forward across the ranks of a process group
  kda_chunk_fwd_seqpar  one GPU, every sequence cut into segments run in parallel
  kda_short_conv, kda_output_gate   layer prologue / epilogue around the core

PyTorch is used for device memory and streams only; every step runs in the
library's CUDA kernels.
"""
from ._lib import (ALGOS, EXPORTS, KdaError, kda_chunk_bwd, kda_chunk_fwd, kda_compose,
                   kda_device_status, kda_output_gate, kda_short_conv, kda_status_string, kda_step,
                   kda_version, library_path, load)
from .autograd import kda_chunk
from .kcp import kcp_chunk_fwd, kda_chunk_fwd_seqpar, seq_segments

__all__ = ["kda_chunk_fwd", "kda_chunk_bwd", "kda_chunk", "kda_step", "kda_compose", "kcp_chunk_fwd",
           "kda_chunk_fwd_seqpar", "seq_segments", "kda_short_conv",
           "kda_output_gate", "kda_device_status",
           "kda_status_string", "kda_version", "KdaError", "ALGOS", "EXPORTS",
           "library_path", "load"]
