"""B200-native (sm_100a) Dynamic Cache Updating for masked-diffusion LLMs.

``dcu`` is the thin binding of ``libdcu.so`` (include/dcu.h); ``inputs`` is the
seeded synthetic-input generator shared by tests and bench; ``build`` compiles
the CUDA sources for sm_100a.
"""
