"""B200-native group-wise affine W4 g64 quantized linear layer.

Python binding of the C ABI declared in include/qlinear.h: argument
marshalling only.  Every step of the computation runs in the CUDA kernels of
libqlinear.so; there is no CPU fallback and no other backend.  Importing this
package does not load the library; the first call does, and fails loudly if
the library is missing or no GPU is visible.

Tensors follow the ABI layout:
    x       torch.bfloat16 [M][K]
    codes   torch.int32    [N][K/8]   (uint32 bit patterns, 8 codes per word, low nibble first)
    scales  torch.float16  [N][K/64]
    biases  torch.float16  [N][K/64]
    y       torch.bfloat16 [M][N]     (y = x . W^T, W[n][k] = scale * code + bias)
The 8-bit variant (forward8, dequant8, pack8, workspace_size8) takes codes as
torch.int32 [N][K/4] (4 codes per word, low byte first) with the same scales
and biases.  swiglu(x, gate, up) runs a SwiGLU up/gate pair of two packed
[I][K] weights in one call: h = silu(x . W_gate^T) * (x . W_up^T).
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    GROUP,
    PATH_AUTO,
    PATH_GEMV,
    PATH_TC_FUSED,
    PATH_TC_SKINNY,
    QLinearError,
    STATUS,
    dequant,
    dequant8,
    device_status,
    forward,
    forward8,
    forward_noalloc,
    last_dispatch,
    lib,
    library_path,
    load_library,
    pack,
    pack8,
    reduce_partials,
    selftest_bounded_wait,
    set_profile_events,
    swiglu,
    swiglu_workspace_size,
    version,
    workspace_size,
    workspace_size8,
)
