"""Four Over Six (4/6) NVFP4 block quantization for B200 (sm_100a).

The kernels live in libfos.so (C ABI in include/fos.h); ``fos`` is the thin
ctypes binding that passes torch device buffers and the current stream to it;
``linear`` orders its calls into a quantized Linear layer's three GEMMs;
``host`` pipelines a batch from and to pinned host memory around them.
"""
from .fos import (  # noqa: F401
    FLAG_RHT16, FLAG_RHT16_COL, FLAG_SCALE_SWIZZLED, STATUS_NONFINITE, STATUS_TIMEOUT, FosError, Options,
    QTensor, amax, dequantize, fake_quantize, gemm_nvfp4, gemm_workspace_size, lib, quantize, scales_size,
    status_string, version,
    workspace_size,
)
from .host import HostQuantizer  # noqa: F401
from .linear import QuantizedWeight, linear_backward, linear_forward, quantize_weight  # noqa: F401
