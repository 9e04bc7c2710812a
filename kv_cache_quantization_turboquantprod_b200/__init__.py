"""TurboQuant-prod KV-cache compression and compressed-KV decode attention on
NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``libtq.so`` (include/tq.h, sources in
``csrc/``); ``tq`` is its thin ctypes binding and ``workloads`` draws the
seeded synthetic inputs.
"""

__all__ = ["tq", "workloads", "build"]
