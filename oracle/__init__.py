"""CPU oracle for block-scaled FP8 / MXFP8 / NVFP4 quantisation (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The GPU library never does.
"""
