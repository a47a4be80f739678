"""libmoe: the Mixture-of-Experts layer hot path on one B200 (sm_100a).

route (top-k or expert choice) -> permute (capacity, expert- or group-major)
-> grouped expert MLPs (tcgen05 tensor cores) -> gate-weighted combine, plus
the co-selection and layer-transition routing statistics.  The kernels live
in ``libmoe.so`` behind the C ABI of ``include/libmoe.h``; ``libmoe`` is its
Python binding and ``layer`` chains the calls into one layer.
"""
