"""B200-native (sm_100a) forward pass of a Mixture-of-Experts FFN layer.

The compute lives in ``libmoe_b200.so`` (CUDA kernels behind a C ABI, declared
in ``include/moe.h``); :mod:`.binding` marshals arguments to it.  Importing the
package itself loads nothing, so :mod:`.inputs` can be used on hosts without a
GPU.
"""
