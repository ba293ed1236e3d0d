"""B200 (sm_100a) implementation of the Kalman Delta Network layer forward.

The compute path is the C-ABI library ``libkdn.so`` (hand-written CUDA, see
``include/kdn.h``); ``kalman_filter_linear_b200.kdn`` is a thin ctypes binding
over it that passes PyTorch tensors' device pointers and the current CUDA
stream.  PyTorch is used only for device memory and streams.  The library is
loaded on first use; if it is missing the call raises instead of falling back.
"""
