"""BitNet b1.58 BitLinear forward on B200 (sm_100a).

The compute lives in ``libbitlinear.so`` (hand-written CUDA behind a C ABI,
declared in ``include/bitlinear.h``); ``ternary_quantized_linear_bitlinear_b200.api``
marshals device pointers into it.  Importing this package does not load the
library; ``api`` does, and raises if it is missing -- there is no CPU path.
"""
