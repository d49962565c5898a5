"""B200-native Kimi Delta Attention (KDA): the gated delta rule's hot path.

The compute lives in ``libkda.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/kda.h``); :mod:`gated_delta_rule_155_b200.kda` is the thin
ctypes binding with the same entry-point names.  Importing the package does not
load the library; the first use of an entry point does, and fails loudly when the
library is missing — there is no CPU fallback.
"""

__all__ = ["forward_chunked", "decode_step", "layer_forward", "KdaError"]


def __getattr__(name):
    if name in __all__:
        from . import kda

        return getattr(kda, name)
    raise AttributeError(name)
