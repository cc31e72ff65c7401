"""ARL2 hybrid attention on B200 (sm_100a).

``workloads`` draws the seeded synthetic inputs; ``arl2`` is the thin ctypes
binding over the C ABI of ``libarl2.so`` (declared in include/arl2.h).
"""
