"""Pins of the oracle's Langevin integrator and of its noise generator (CPU only).

  - Philox4x32-10 against the known-answer vectors published with the generator
    (Salmon, Moraes, Dror and Shaw, 2011; Random123 distribution);
  - Box-Muller deviates: mean 0, variance 1, no correlation between components;
  - friction 0: the O step is the identity and BAOAB reduces exactly to velocity Verlet;
  - free particles thermalise: <KE> per degree of freedom = kB T / 2, and the velocity
    autocorrelation decays as exp(-friction t).
"""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth


@pytest.mark.parametrize("ctr,key,expect", [
    ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
    ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
    ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
     [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
])
def test_philox_known_answers(oracle, ctr, key, expect):
    assert oracle.philox4x32_10(ctr, key).tolist() == expect


def test_noise_is_standard_normal(oracle):
    xi = np.array([oracle.langevin_noise(1234, s, i) for s in range(200) for i in range(150)])
    n = len(xi)
    assert np.all(np.abs(xi.mean(0)) < 5 / np.sqrt(n))
    assert np.all(np.abs(xi.var(0) - 1.0) < 5 * np.sqrt(2.0 / n))
    c = np.corrcoef(xi.T)
    assert np.all(np.abs(c[np.triu_indices(3, 1)]) < 5 / np.sqrt(n))
    # distinct streams for distinct seeds / steps / atoms
    assert not np.allclose(oracle.langevin_noise(1, 0, 0), oracle.langevin_noise(2, 0, 0))
    assert not np.allclose(oracle.langevin_noise(1, 0, 0), oracle.langevin_noise(1, 1, 0))
    assert not np.allclose(oracle.langevin_noise(1, 0, 0), oracle.langevin_noise(1, 0, 1))


def test_zero_friction_is_velocity_verlet(oracle):
    w = synth.make_workload(1)
    v0 = synth.maxwell_boltzmann(32, 1, 12.0, 300.0, 4001).astype(np.float64)
    p1, v1, f1, e1, k1, _ = oracle.md_vv(w.model, w.weights, w.system, w.pos, v0, w.types, 12.0, 2.0, 15)
    p2, v2, f2, e2, k2 = oracle.md_langevin(w.model, w.weights, w.system, w.pos, v0, w.types, 12.0, 2.0, 15,
                                            300.0, 0.0, seed=7)
    np.testing.assert_allclose(p2, p1, rtol=0, atol=1e-11)
    np.testing.assert_allclose(v2, v1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(e2, e1, rtol=1e-12)


def test_free_particles_thermalise(oracle):
    """Zero the filter output so that forces vanish: the O step alone drives the velocities,
    whose stationary distribution has <v^2> = kB T kappa / m per component, and whose
    correlation with the initial velocities decays as exp(-friction t)."""
    F, K, T, nt = 8, 4, 1, 2
    model = synth.ModelCfg(F=F, K=K, T=T, n_types=nt, r_cut=5.0)
    blob = synth.weights_blob(F, K, T, nt, seed=3, bias_std=0.1)
    p = nt * F + F * K + F
    blob[p:p + F * F + F] = 0.0
    system = synth.SystemCfg(64, 4)
    w = synth.make_custom(model, system, 9, "rw")
    mass, temp, friction, dt = 12.0, 300.0, 0.01, 4.0
    v0 = np.full((256, 3), 0.02)
    _, v, _, _, ekin = oracle.md_langevin(model, blob, system, w.pos, v0, w.types, mass, dt, 400, temp, friction, seed=11)
    sigma2 = synth.KB * temp * synth.KAPPA / mass
    assert abs(v.var() / sigma2 - 1.0) < 5 * np.sqrt(2.0 / v.size)
    # KE of the last 200 steps averages (3/2) n kB T per replica
    ke_mean = ekin[200:].mean()
    assert abs(ke_mean / (1.5 * 64 * synth.KB * temp) - 1.0) < 0.05
    # one step from a fixed velocity: mean a v0, spread b (exact O-step law, no force)
    _, v1, _, _, _ = oracle.md_langevin(model, blob, system, w.pos, v0, w.types, mass, dt, 1, temp, friction, seed=12)
    a = np.exp(-friction * dt)
    b = np.sqrt((1 - a * a) * sigma2)
    xi = np.array([oracle.langevin_noise(12, 0, i) for i in range(256)])
    np.testing.assert_allclose(v1, a * v0 + b * xi, rtol=0, atol=1e-15)
