"""B200 (sm_100a) Lightning Attention: prefill and decode behind a C ABI.

Importing the package loads nothing; the CUDA library is loaded on the first
call of a function in ``long_context_fwd_b200.ops`` and a missing library
raises instead of falling back to any other implementation (build it with
``python -m long_context_fwd_b200.build``).
"""
__all__ = ["inputs", "ops"]
