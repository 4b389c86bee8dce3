"""Single-device Megatron-style tensor-parallel transformer layer for B200.

The compute path is the C-ABI library ``libtpl.so`` (hand-written CUDA for
sm_100a); ``tpl`` is its thin ctypes binding and ``synth`` draws seeded
synthetic inputs.  Importing this package loads nothing; importing ``tpl``
loads the library and fails loudly if it has not been built.
"""
__all__ = ["tpl", "synth"]
