"""Causal Lightning Attention on B200 (sm_100a): chunked prefill and decode step.

The compute path is a C-ABI CUDA library (``liblightning_b200.so``, declared in
``include/la.h``).  This package is its thin Python binding: argument
marshalling from torch tensors to device pointers, nothing else.  Importing the
package does not load the library; the first call does, and fails loudly when
the library has not been built.
"""
from .api import (  # noqa: F401
    LAError,
    la_backward,
    la_decode_step,
    la_decode_steps,
    la_device_status,
    la_forward,
    la_forward_f32,
    la_forward_host,
    la_forward_state,
    la_segment_state,
    la_state_prefix,
    la_status_string,
    library_path,
    load_library,
)
