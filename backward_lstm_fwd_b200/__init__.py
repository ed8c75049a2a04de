"""liblstm: B200-native single-layer LSTM forward pass and BPTT.

The compute lives in the C-ABI shared library ``liblstm.so`` (hand-written
sm_100a CUDA kernels); ``backward_lstm_fwd_b200.binding`` is its thin ctypes
binding.  Import that module explicitly; importing the package alone loads no
native code.
"""
