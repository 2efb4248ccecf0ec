"""Blocked-Shampoo optimizer step for the NVIDIA B200 (sm_100a).

The compute lives in ``libshampoo.so`` (C ABI, include/shampoo.h); this
package holds its ctypes binding (``binding``), the step orchestrator
(``optimizer``), the seeded synthetic inputs (``workloads``) and the build
script (``build``).  Importing the package loads nothing; the library is
loaded on first use.
"""
__all__ = ["binding", "optimizer", "workloads", "build"]
