"""B200-native stochastic-computing (SC) bipolar XNOR matmul.

The compute lives in the sm_100a CUDA library ``libsc_b200.so`` behind the C
ABI of ``include/sc.h``; ``_lib`` is its ctypes binding and ``sc`` adds torch
device buffers and the full quantise -> assign rows -> count + decode step.
``workloads`` draws the seeded synthetic inputs.
"""
from ._lib import (EXPORTS, ScError, ScMatmulDesc, load, sc_assign_rows, sc_build_table,  # noqa: F401
                   sc_kband_tilt, sc_last_error, sc_matmul, sc_quantize, sc_table_destroy,
                   sc_table_info, sc_version, sc_matmul_engine)

__all__ = ["EXPORTS", "ScError", "ScMatmulDesc", "load", "sc_assign_rows", "sc_build_table",
           "sc_kband_tilt", "sc_last_error", "sc_matmul", "sc_quantize", "sc_table_destroy",
           "sc_table_info", "sc_version", "sc_matmul_engine"]
