"""AdaFuse adapter switch for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libadafuse.so`` (C ABI in ``include/adafuse.h``).
Every step of the hot path -- pre-gating and the fused switch -- runs in the
library's CUDA kernels; this package only marshals arguments.  PyTorch is
used by callers for device memory and streams.  There is no CPU fallback:
importing the binding fails loudly when the compiled library is missing.
"""
from .binding import (  # noqa: F401
    ADAFUSE_OK, ADAFUSE_ERR_INVALID_ARG, ADAFUSE_ERR_UNSUPPORTED_SHAPE, ADAFUSE_ERR_CUDA,
    ADAFUSE_ERR_DEVICE_FAULT, ADAFUSE_ERR_UNSUPPORTED_DEVICE, ADAFUSE_ERR_OUT_OF_MEMORY,
    ADAFUSE_STATUS_BAD_EXPERT, ADAFUSE_STATUS_BAD_GATE, ADAFUSE_STATUS_TIMEOUT,
    ADAFUSE_KERNEL_AUTO, ADAFUSE_KERNEL_MMA_SYNC, ADAFUSE_KERNEL_TCGEN05, AdafuseError, Route, Target, Desc,
    lib, library_path, adafuse_create, adafuse_destroy, adafuse_pregate, adafuse_switch,
    adafuse_switch_batch_layers, adafuse_get_device_status, adafuse_set_switch_kernel,
    adafuse_get_switch_kernel, adafuse_segment_table, adafuse_set_base, adafuse_rebase,
    adafuse_rebase_layers,
    adafuse_tile_size, adafuse_strerror, adafuse_last_error, Switcher,
)
