"""Pins of the oracle's velocity-Verlet integrator (CPU only).

  - free flight: with the second filter layer zeroed the forces vanish, so r(t) = r0 + t v0;
  - time reversibility: n steps, flip v, n steps returns to r0 (velocity Verlet is
    symmetric in time);
  - second order: the total-energy error of a fixed time span scales as dt^2.
"""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth


def test_free_flight(oracle):
    F, K, T, nt = 8, 4, 2, 3
    model = synth.ModelCfg(F=F, K=K, T=T, n_types=nt, r_cut=6.0)
    blob = synth.weights_blob(F, K, T, nt, seed=12, bias_std=0.3)
    p = nt * F
    for t in range(T):
        p += F * K + F
        blob[p:p + F * F + F] = 0.0
        p += F * F + F + 2 * (F * F + F)
    system = synth.SystemCfg(10, 2)
    w = synth.make_custom(model, system, 3)
    v0 = synth.maxwell_boltzmann(10, 2, 12.0, 300.0, seed=5).astype(np.float64)
    n, dt = 25, 2.0
    pos, vel, forces, epot, ekin, _ = oracle.md_vv(model, blob, system, w.pos, v0, w.types, 12.0, dt, n)
    np.testing.assert_allclose(pos, w.pos.astype(np.float64) + n * dt * v0, rtol=0, atol=1e-10)
    np.testing.assert_allclose(vel, v0, rtol=0, atol=0)
    assert np.all(forces == 0.0)
    ke0 = 0.5 * 12.0 * (v0.reshape(2, 10, 3) ** 2).sum(axis=(1, 2)) / synth.KAPPA
    np.testing.assert_allclose(ekin[-1], ke0, rtol=1e-12)


def test_time_reversible(oracle):
    w = synth.make_workload(1)
    v0 = synth.maxwell_boltzmann(32, 1, 12.0, 300.0, seed=4001).astype(np.float64)
    n, dt = 30, 2.0
    pos, vel, forces, *_ = oracle.md_vv(w.model, w.weights, w.system, w.pos, v0, w.types, 12.0, dt, n)
    pos2, vel2, *_ = oracle.md_vv(w.model, w.weights, w.system, pos, -vel, w.types, 12.0, dt, n, forces=forces)
    np.testing.assert_allclose(pos2, w.pos.astype(np.float64), rtol=0, atol=1e-9)
    np.testing.assert_allclose(-vel2, v0, rtol=0, atol=1e-12)


def test_energy_error_is_second_order(oracle):
    """Max |E_tot(t) - E_tot(0)| over the same 200 fs at dt and dt/2: ratio near 4."""
    w = synth.make_workload(1)
    v0 = synth.maxwell_boltzmann(32, 1, 12.0, 300.0, seed=4001).astype(np.float64)
    rp, cl = oracle.neighbors(w.system, w.model.r_cut, w.pos)
    E0, F0, _ = oracle.energy_forces(w.model, w.weights, w.system, w.pos, w.types, rp, cl)
    ke0 = 0.5 * 12.0 * (v0 ** 2).sum() / synth.KAPPA
    errs = []
    for dt in (8.0, 4.0, 2.0):
        n = int(round(200.0 / dt))
        _, _, _, epot, ekin, _ = oracle.md_vv(w.model, w.weights, w.system, w.pos, v0, w.types,
                                              12.0, dt, n, forces=F0)
        etot = epot[:, 0] + ekin[:, 0]
        errs.append(np.abs(etot - (E0[0] + ke0)).max())
    assert errs[0] > 0
    r1, r2 = errs[0] / errs[1], errs[1] / errs[2]
    assert 3.0 < r1 < 5.3 and 3.0 < r2 < 5.3, (errs, r1, r2)
