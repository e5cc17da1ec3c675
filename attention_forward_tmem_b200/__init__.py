"""B200 (sm_100a) attention forward: tcgen05/TMEM flash kernel behind a C ABI.

The public calls live in :mod:`attention_forward_tmem_b200.api`; they marshal
torch tensors into the C ABI declared in ``include/wf_attn.h`` and run every
step in the CUDA library ``libwfattn.so``.  There is no CPU path: if the
library is missing or no sm_100 device is present, the calls raise.

Importing the package does not load the library; the first API call does.
"""
__all__ = ["attn_fwd", "scaled_dot_product_attention", "merge", "dca", "BlockKVCache", "device_status",
           "MaskType", "WfError"]


def __getattr__(name):
    if name in __all__:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
