"""B200 (sm_100a) quantised MoE layer: C-ABI library libmoeq.so + binding.

Submodules: ``moeq`` (ctypes binding, one function per C entry point),
``layer`` (a layer driven call by call through the ABI), ``inputs`` (seeded
synthetic inputs), ``build`` (nvcc build of the library).  Importing the
package loads nothing; ``moeq.load()`` opens the library and refuses to run
without a CUDA device.
"""
