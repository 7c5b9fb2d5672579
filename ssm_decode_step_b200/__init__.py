"""Quantized recurrent-state decode step on B200 (sm_100a).

The product is the CUDA library libqstate.so (C ABI in include/qstate.h);
this package holds its sources (csrc/), its build step (build.py), a thin
ctypes binding (qstate.py) and the seeded synthetic workloads
(workloads.py).
"""
from .qstate import (Config, HostPipeline, QState, QStateError, decode_step, init, query_sizes,
                     readout, status_string)

__all__ = ["Config", "HostPipeline", "QState", "QStateError", "decode_step", "init", "query_sizes",
           "readout", "status_string"]
