"""MLA decoding over a paged latent KV cache, as a C-ABI library for B200 (sm_100a).

The compute path lives in `csrc/` (CUDA kernels behind an extern "C" boundary
declared in `include/mla_decode.h`); `binding` marshals torch tensors into that
boundary.  Importing this package does not load the library; `binding` does.
"""

__all__ = ["binding", "synth"]
