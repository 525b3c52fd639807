"""Block-GTQ / TQ-MSE packed-KV decode attention for NVIDIA B200 (sm_100a).

The compute lives in ``libbgtq.so`` (hand-written CUDA behind a C ABI declared in
``include/bgtq.h``); ``binding`` marshals arguments to it. ``synth`` draws seeded
synthetic inputs.
"""
__all__ = ["binding", "synth"]
