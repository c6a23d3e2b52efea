"""B200-native VSA-style block-sparse video attention (forward pass).

The compute path lives in the shared library ``libvsa.so`` (C ABI declared in
``include/vsa.h``) built from ``csrc/`` for sm_100a. ``vsa`` is its thin
ctypes binding; importing this package does not load the library, the first
call does, and it raises if the library is missing.
"""

__all__ = ["vsa", "workloads"]
