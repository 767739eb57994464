"""csffn: contextually sparse gated FFN at decode time on B200 (sm_100a).

The compute path is libcsffn.so (hand-written CUDA, C ABI in include/csffn.h);
``binding`` marshals torch tensors into it.  ``synth`` holds the seeded
synthetic workloads and ``offline`` the host-side SVD factorisation.
"""
from ._abi import (ACT_RELU, ACT_SILU, BF16, CAL_GLOBAL_ABS_ACT, CAL_PER_NEURON_PRED,  # noqa: F401
                   CAL_PER_NEURON_RECALL, F32, OUT_BF16, OUT_F32, OUT_F32_ACCUMULATE, CsffnError)

__all__ = ["binding", "synth", "offline"]
