"""B200-native forward pass of a Mixture-of-Experts SwiGLU FFN layer.

The compute path lives in ``libmoe_b200.so`` (hand-written CUDA for sm_100a
behind a C ABI, see ``include/moe.h``).  ``binding`` marshals torch tensors
into that ABI; ``synth`` draws seeded synthetic inputs.  Importing this
package does not load the library: ``binding`` does, and fails loudly when
the library is missing.
"""
__all__ = ["binding", "synth"]
