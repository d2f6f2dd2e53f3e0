"""B200 (sm_100a) native-sparse-attention layer of LSRM behind a C ABI.

`nsa` is the thin ctypes binding of liblsrm_nsa.so (include/lsrm_nsa.h);
`build` compiles the library in-tree with nvcc.
"""
from . import nsa  # noqa: F401
