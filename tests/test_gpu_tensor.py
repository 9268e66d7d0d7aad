"""Tensor-core (tcgen05) precisions vs the CPU oracle, through the C ABI.

SN_PREC_TC32 (fp16 two-term split, fp32-accurate) must meet the fp32 tolerance of
tests/test_gpu_parity.py: |err| <= 1e-5 * max(1, RMS) + 1e-4 |ref| per element.

SN_PREC_FP16 (single fp16 operands, fp32 accumulation; the pages' W16A16) must meet
|err| <= 5e-3 * |ref| + 5e-3 * RMS(ref) per element: 5e-3 relative, with the absolute part on
the scale of the quantity, because fp16 rounding of the operands (2^-11 relative) produces
errors proportional to the magnitude of the summed terms, not of each component.
"""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth
from tests.test_gpu_parity import assert_close, report, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PREC_FP16, PREC_TC32, PREC_FP16_CH = 1, 2, 3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def assert_close16(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    bound = 5e-3 * np.abs(ref) + 5e-3 * float(np.sqrt(np.mean(ref ** 2)))
    report(what, gpu, ref, bound, "fp16: 5e-3 |ref| + 5e-3 RMS")
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                           f"max err/bound {(err / bound).max():.3g}")


def run(oracle, w, dev, precision):
    from schnet_gnn_molecular_cell_b200 import Context
    s, m = w.system, w.model
    ctx = Context(m, w.weights, precision=precision)
    rp, cl = oracle.neighbors(s, m.r_cut, w.pos, "cells" if s.periodic else "brute")
    E_o, F_o, _ = oracle.energy_forces(m, w.weights, s, w.pos, w.types, rp, cl)
    E_g, F_g = ctx.energy_forces(s, to_dev(w.pos, dev), to_dev(w.types, dev), to_dev(rp, dev), to_dev(cl, dev))
    ctx.sync()
    return ctx, E_g.cpu().numpy(), F_g.cpu().numpy(), E_o, F_o


CASES = [
    ("cfg2", lambda: synth.make_workload(2)),
    ("cfg4", lambda: synth.make_workload(4)),
    ("ragged_chains_bias", lambda: synth.make_custom(synth.ModelCfg(128, 50, 3, 20, 12.0), synth.SystemCfg(37, 5), 501, "saw", bias_std=0.2)),
    ("k20_T1", lambda: synth.make_custom(synth.ModelCfg(128, 20, 1, 3, 9.0, 2.5), synth.SystemCfg(70, 2), 503, "rw", bias_std=0.1)),
    ("box_replicas", lambda: synth.make_custom(synth.ModelCfg(128, 50, 3, 8, 5.0), synth.SystemCfg(300, 3, (16.0, 16.0, 16.0)), 507, "box", bias_std=0.1)),
    ("one_atom_replicas", lambda: synth.make_custom(synth.ModelCfg(128, 50, 2, 8, 5.0), synth.SystemCfg(1, 7), 508, "rw", bias_std=0.2)),
]


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_tc32_matches_oracle_at_fp32_tolerance(oracle, dev, name, mk):
    _, E_g, F_g, E_o, F_o = run(oracle, mk(), dev, PREC_TC32)
    assert_close(E_g, E_o, "energy")
    assert_close(F_g, F_o, "forces")


@pytest.mark.parametrize("precision", [PREC_FP16, PREC_FP16_CH], ids=["fp16", "fp16_ch"])
@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_fp16_matches_oracle_at_fp16_tolerance(oracle, dev, name, mk, precision):
    """Both 16-bit modes: weights cast as they are, and weights stored per output channel as
    W / max|W| with the scale applied in fp32 (FlashSchNet §4.4)."""
    _, E_g, F_g, E_o, F_o = run(oracle, mk(), dev, precision)
    assert_close16(E_g, E_o, "energy")
    assert_close16(F_g, F_o, "forces")



def test_tc32_config5(oracle, dev):
    _, E_g, F_g, E_o, F_o = run(oracle, synth.make_workload(5), dev, PREC_TC32)
    assert_close(E_g, E_o, "energy")
    assert_close(F_g, F_o, "forces")


def test_fp16_config5(oracle, dev):
    # every force component of the 65,536-atom box (2.1 M edges) in the fp16-operand mode
    _, E_g, F_g, E_o, F_o = run(oracle, synth.make_workload(5), dev, PREC_FP16)
    assert_close16(E_g, E_o, "energy")
    assert_close16(F_g, F_o, "forces")


@pytest.mark.parametrize("precision", [PREC_FP16, PREC_TC32])
def test_tensor_modes_bitwise_deterministic_and_md(oracle, dev, precision):
    from schnet_gnn_molecular_cell_b200 import Context
    w = synth.make_workload(4)
    ctx = Context(w.model, w.weights, precision=precision)
    pos = to_dev(w.pos, dev)
    types = to_dev(w.types, dev)
    rp, cl = ctx.neighbors(w.system, pos)
    E1, F1 = ctx.energy_forces(w.system, pos, types, rp, cl)
    E1, F1 = E1.clone(), F1.clone()
    E2, F2 = ctx.energy_forces(w.system, pos, types, rp, cl)
    ctx.sync()
    assert torch.equal(E1, E2) and torch.equal(F1, F2)
    vel = to_dev(synth.maxwell_boltzmann(4096, 1, 12.0, 300.0, 4004), dev)
    e = torch.empty(1, device=dev)
    k = torch.empty(1, device=dev)
    ctx.md_step(w.system, pos, vel, F1, types, 12.0, 2.0, 3, e, k)
    ctx.sync()
    assert torch.isfinite(e).all() and torch.isfinite(F1).all()


def test_tensor_modes_need_f128():
    from schnet_gnn_molecular_cell_b200 import Context, SNError, Status
    m = synth.ModelCfg(64, 32, 2, 4, 10.0)
    with pytest.raises(SNError) as ei:
        Context(m, synth.weights_blob(64, 32, 2, 4, seed=1), precision=PREC_TC32)
    assert ei.value.status == Status.UNSUPPORTED
