"""B200-native generalized delta-rule matrix memory (chunked forward and decode step).

The compute lives in ``libgdr.so`` (CUDA kernels for sm_100a behind the C ABI in
``include/gdr.h``); ``matrix_memory_rnn_b200.gdr`` is its Python binding and
``matrix_memory_rnn_b200.synth`` the seeded input generator.
"""
