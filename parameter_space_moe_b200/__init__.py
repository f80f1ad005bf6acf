"""B200-native (sm_100a) forward pass of the Swimba (Switch Mamba) token-mixer layer.

The compute path is libswimba.so (hand-written CUDA behind the C ABI in include/swimba.h); the
`swimba` module is its ctypes binding.  Importing the package itself loads nothing, so the input
generator and workload table can be used on machines without a GPU.
"""
