"""B200-native persistent decode megakernel.

The product is the C-ABI library ``libmk.so`` (declared in include/mk.h) and
its thin ctypes binding :mod:`persistent_decode_megakernel_02_b200.mk`.
:mod:`persistent_decode_megakernel_02_b200.workloads` holds the model shapes
and seeded synthetic inputs.
"""
