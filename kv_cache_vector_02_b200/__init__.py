"""B200-native TurboQuant-style KV-cache compression (libtq) and its binding.

The compute path is the CUDA library ``libtq.so`` built from ``csrc/``; this
package only marshals arguments to it (``tq``) and generates seeded synthetic
workloads (``workloads``).  Importing ``tq`` fails loudly when the library has
not been built.
"""

__all__ = ["tq", "workloads", "build"]
