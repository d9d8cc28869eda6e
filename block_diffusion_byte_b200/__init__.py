"""B200-native engine for the Fast-BLT local-decoder step.

* ``binding``  -- ctypes binding of the C ABI in include/bltdec.h
* ``driver``   -- host-side generation loops (BLT-D, BLT-S, BLT-DV, AR greedy)
                  over the C ABI, with the synthetic patcher / latents of
                  :mod:`workload` standing in for the entropy model, encoder
                  and global transformer
* ``_build``   -- nvcc build of libbltdec.so (sm_100a)
"""

from . import binding  # noqa: F401
