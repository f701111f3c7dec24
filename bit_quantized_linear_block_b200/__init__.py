"""B200-native quantized linear layer: block Hadamard + NVFP4/INT8 activation
quantization routed by DMPQ's Gamma, NVFP4 / Q-ARVD dual-scale weights, and
tcgen05 GEMMs.  The compute lives in ``libqlinear.so`` (CUDA, sm_100a); the
Python module ``qlinear`` is a thin ctypes binding over its C ABI.

Import ``bit_quantized_linear_block_b200.qlinear`` for the binding; this
package ``__init__`` loads nothing so that host-only helpers stay importable
on machines without a GPU."""
