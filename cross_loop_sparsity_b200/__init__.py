"""B200-native lazy-update looped-Transformer inference (FlashLoop).

The library is ``libflashloop.so`` (C ABI, declared in ``include/flashloop.h``);
``cross_loop_sparsity_b200.flashloop`` is its ctypes binding.  Nothing is
loaded at import time: ``synth`` (seeded inputs) works without a GPU.
"""
