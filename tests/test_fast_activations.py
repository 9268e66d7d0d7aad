"""The fp16-operand mode's shifted softplus replaces log1p(u), u in [0, 1], by a degree-5
polynomial (Chebyshev interpolation at the first-kind nodes).  Its coefficients are read from
the CUDA header and checked here against log1p in double precision: the kernels' error bound
(1.1e-5 absolute, far below the 2^-11 relative rounding of the fp16 operand it feeds) holds.
The tanh-based sigmoid uses the hardware tanh and is covered by the GPU parity tests."""
import re
from pathlib import Path

import numpy as np

HDR = Path(__file__).resolve().parents[1] / "schnet_gnn_molecular_cell_b200" / "csrc" / "sn_tc_common.cuh"


def _coefficients():
    text = HDR.read_text()
    c = {int(k): float(v) for k, v in re.findall(r"constexpr float LOG1P_C(\d) = ([-+0-9.eE]+)f;", text)}
    assert sorted(c) == list(range(6)), "six coefficients LOG1P_C0..C5 expected"
    return np.array([c[k] for k in range(6)], dtype=np.float32)


def test_log1p_polynomial_error_bound():
    c = _coefficients()
    u = np.linspace(0.0, 1.0, 100001, dtype=np.float32)
    p = np.full_like(u, c[5])
    for k in (4, 3, 2, 1, 0):          # Horner in float32 with fused multiply-add semantics
        p = (p.astype(np.float64) * u + c[k]).astype(np.float32)
    err = np.abs(p.astype(np.float64) - np.log1p(u.astype(np.float64)))
    assert err.max() < 1.5e-5


def test_ssp_from_polynomial_matches_definition():
    c = _coefficients().astype(np.float64)
    x = np.linspace(-20.0, 20.0, 40001)
    u = np.exp(-np.abs(x))
    p = np.polynomial.polynomial.polyval(u, c)
    ssp = np.maximum(x, 0.0) + p - np.log(2.0)
    ref = np.log(0.5 * np.exp(x) + 0.5)     # ssp(x) = ln(e^x / 2 + 1 / 2)
    assert np.max(np.abs(ssp - ref)) < 1.5e-5
