"""B200-native NVFP4 quantized linear-layer training path.

The compute lives in the CUDA library libnvfp4.so (C ABI, include/nvfp4.h);
`nvfp4_bit_quantized_amax_b200.capi` is its thin Python binding.  Importing
this package does not load the library; `capi.load()` does, and raises if the
library is missing -- there is no CPU fallback.
"""
