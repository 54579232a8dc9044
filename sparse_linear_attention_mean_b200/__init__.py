"""RoLA hybrid sparse + linear attention for video DiTs, native on B200 (sm_100a).

The compute path lives in ``librola.so`` (hand-written CUDA for sm_100a behind
a C ABI, declared in ``include/rola.h``); ``binding`` marshals torch tensors
into it.  ``synth`` draws the seeded synthetic workloads.
"""
__all__ = ["binding", "synth"]
