"""B200-native fused top-k Mixture-of-Experts layer.

The compute path lives in the CUDA library ``libmoe_b200.so`` (sources in
``csrc/``, C ABI in ``include/moe_b200.h``); :mod:`moe_layer_top_b200.ops`
is the thin ctypes binding over it.  The library is loaded on first use and a
missing or unloadable library raises: there is no CPU fallback.
:mod:`moe_layer_top_b200.expert_parallel` runs the layer sharded by expert over
a ``torch.distributed`` process group (NCCL, or the library's fused combine +
all-reduce over peer memory).
"""

__all__ = ["ops", "inputs", "expert_parallel"]
