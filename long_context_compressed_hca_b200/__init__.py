"""B200-native hybrid compressed attention (DeepSeek-V4 CSA + HCA).

The compute path is the C-ABI library libhca.so (hand-written sm_100a CUDA);
`binding` is a thin ctypes layer over it.  Importing the package does not load
the library; `binding.lib()` does, and raises if it is missing.
"""
__all__ = ["binding", "synth", "workloads"]
