"""Quantized recurrent-state decode step for gated delta-rule linear attention
(GDN and KDA), B200-native.

``StatePool`` (state.py) is the torch-facing handle over the C ABI in
include/sq.h; ``_abi`` is the raw ctypes binding; ``synth`` draws seeded
synthetic workloads. The compute runs in libsq.so (csrc/), built in-tree by
``build.py`` for sm_100a.
"""
from . import _abi  # noqa: F401
from ._abi import (SQ_FMT_FP32, SQ_FMT_PACKED, SQ_GATE_HEAD, SQ_GATE_KEY_CHANNEL,  # noqa: F401
                   SQ_STATUS_BAD_SLOT, SQ_STATUS_NAN, SQ_STATUS_SATURATED, SQ_STATUS_TIMEOUT, SQError)


def __getattr__(name):
    if name == "StatePool":
        from .state import StatePool
        return StatePool
    raise AttributeError(name)
