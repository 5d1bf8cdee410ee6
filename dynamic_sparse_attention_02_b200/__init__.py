"""B200-native MInference dynamic sparse prefill.

The compute path lives in the C-ABI library ``libminfer.so`` (hand-written
sm_100a CUDA, declared in ``include/minfer.h``); ``binding`` is a thin ctypes
layer over it.  ``synth`` draws the seeded synthetic inputs.  Importing this
package does not load the CUDA library; the first call through ``binding``
does, and it raises if the library is missing.
"""

__all__ = ["binding", "synth"]
