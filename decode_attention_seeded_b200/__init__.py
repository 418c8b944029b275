"""B200-native TurboQuant-style compressed-KV cache: quantize/append and decode attention.

The compute lives in ``libtq.so`` (C ABI declared in ``include/tq.h``; CUDA
kernels for sm_100a). ``binding`` marshals torch tensors into those calls;
``synth`` holds the seeded synthetic workloads. Importing this package does not
load the library; ``binding.lib()`` does, and raises if it is missing.
"""

__all__ = ["binding", "synth"]
