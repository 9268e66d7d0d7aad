"""B200 (sm_100a) SchNet energy/force library: neighbour list, fused CFConv energy and
forces, velocity Verlet, behind the C ABI of include/sn.h (libsnflash.so).

    from schnet_gnn_molecular_cell_b200 import Context, synth
"""
from . import synth
from .binding import (Context, SNError, Status, load, version, PREC_FP32, PREC_FP16, PREC_TC32,
                      PREC_FP16_CH)

__all__ = ["Context", "SNError", "Status", "load", "version", "synth", "PREC_FP32", "PREC_FP16", "PREC_TC32",
           "PREC_FP16_CH"]
