"""Diagonal-batched ARMT prefill on B200 (sm_100a): a C-ABI CUDA library and its binding.

The library (librmt.so, API in include/rmt.h) runs the (layer, segment) grid of an
Associative Recurrent Memory Transformer in anti-diagonals, one grouped launch per step.
`rmt` is the ctypes binding; importing it loads the library and fails loudly if it is not
built.
"""
__all__ = ["rmt"]
