"""B200 (sm_100a) Dynamic Linear Attention forward.

``dynamic_state_memory_b200.dla`` is the ctypes binding of libdla.so (the CUDA
path); ``dynamic_state_memory_b200.synth`` draws seeded synthetic inputs.
Importing the package itself loads nothing.
"""
