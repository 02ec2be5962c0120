"""CalibAtt calibrated block-sparse / anchor-row attention for NVIDIA B200 (sm_100a).

The computation lives in libcalibatt.so (C ABI: include/calibatt.h), built
in-tree by ``calibrated_block_sparse_calibatt_b200.build.build()``.  Import
``calibrated_block_sparse_calibatt_b200.calibatt`` for the Python binding; it
loads the library and raises if it has not been built.
"""

__all__ = ["calibatt", "build"]
