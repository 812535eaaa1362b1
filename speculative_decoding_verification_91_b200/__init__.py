"""B200-native speculative-decoding verify step.

The compute path is the CUDA library ``libspecverify.so`` (kernels for
sm_100a behind a C ABI, declared in include/specverify.h); ``binding``
marshals arguments to it through ctypes and ``runtime`` holds device
buffers (PyTorch is used for device memory and streams only).
Importing this package does not load the library; the first call does.
"""
