"""B200 (sm_100a) kernels for Samba's two token mixers behind a C ABI.

``hybrid_ssm_sliding_b200.ops`` holds the Python entry points (thin ctypes
wrappers over libsamba.so); ``workloads`` holds the seeded synthetic inputs.
Importing the package does not load the CUDA library; the first call does.
"""

__all__ = ["ops", "workloads"]
