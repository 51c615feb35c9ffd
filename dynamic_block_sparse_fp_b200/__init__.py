"""FlexPrefill prefill-attention hot path for B200 (sm_100a).

The compute lives in ``libfp.so`` (hand-written CUDA behind a C ABI declared in
``include/fp.h``); ``ops`` is a thin ctypes binding over it.  Importing this
package loads nothing; ``ops`` loads the library on first use and raises if it
is missing.
"""
__all__ = ["ops", "synth"]
