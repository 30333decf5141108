"""SAS gated block-sparse attention for B200 (sm_100a): C-ABI library libsas
(include/sas.h) with a thin ctypes binding (``sas``) and seeded synthetic
workload generators (``workloads``)."""
