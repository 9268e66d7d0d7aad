"""The seeded synthetic inputs have the structure the input recipe states: fixed 3.8 A bonds,
self-avoidance of the SAW chains, uniform positions inside the periodic boxes, bead types in
range, Maxwell-Boltzmann velocities at the requested temperature with no centre-of-mass drift,
and weights with the documented layout and N(0, 1/fan_in) scale."""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth


def test_chain_bonds_and_self_avoidance():
    pos = synth.chains(269, 4, 1234, saw=True).astype(np.float64).reshape(4, 269, 3)
    bonds = np.linalg.norm(np.diff(pos, axis=1), axis=2)
    assert np.allclose(bonds, synth.BOND, atol=1e-4)
    for r in range(4):
        d = np.linalg.norm(pos[r][:, None, :] - pos[r][None, :, :], axis=2)
        off = np.abs(np.subtract.outer(np.arange(269), np.arange(269))) >= 2
        assert d[off].min() >= synth.BOND - 1e-4          # no non-bonded bead closer than a bond
    walk = synth.chains(269, 2, 99, saw=False).astype(np.float64).reshape(2, 269, 3)
    assert np.allclose(np.linalg.norm(np.diff(walk, axis=1), axis=2), synth.BOND, atol=1e-4)


def test_chains_start_at_the_origin_and_are_seeded():
    a = synth.chains(50, 3, 7, saw=True)
    b = synth.chains(50, 3, 7, saw=True)
    assert np.array_equal(a, b)
    assert np.allclose(a.reshape(3, 50, 3)[:, 0, :], 0.0)


@pytest.mark.parametrize("cfg", [4, 5])
def test_box_positions_inside_the_box(cfg):
    w = synth.make_workload(cfg)
    L = np.asarray(w.system.box)
    assert w.pos.dtype == np.float32 and (w.pos >= 0).all() and (w.pos < L).all()
    # uniform: every octant holds about an eighth of the atoms
    octant = ((w.pos >= L / 2) * np.array([1, 2, 4])).sum(axis=1)
    counts = np.bincount(octant, minlength=8) / len(octant)
    assert np.all(np.abs(counts - 0.125) < 0.03)


def test_types_in_range():
    for cfg in (1, 2, 4):
        w = synth.make_workload(cfg)
        assert w.types.min() >= 0 and w.types.max() < w.model.n_types


def test_maxwell_boltzmann_temperature_and_no_drift():
    m, T = 12.0, 300.0
    v = synth.maxwell_boltzmann(269, 64, m, T, 4002).astype(np.float64).reshape(64, 269, 3)
    assert np.allclose(v.mean(axis=1), 0.0, atol=1e-6)
    # equipartition: m <v^2> / (3 kB kappa) = T up to sampling error (3 dof per bead)
    T_est = m * np.mean(np.sum(v ** 2, axis=2)) / (3 * synth.KB * synth.KAPPA)
    assert abs(T_est / T - 1) < 0.02


def test_weight_blob_layout_and_scale():
    F, K, T, nt = 128, 50, 3, 20
    w = synth.weights_blob(F, K, T, nt, 3002)
    assert w.size == synth.n_weights(F, K, T, nt) and w.dtype == np.float32
    W1 = w[nt * F: nt * F + F * K].reshape(F, K)              # first block's filter layer 1
    assert abs(W1.std() * np.sqrt(K) - 1.0) < 0.05            # N(0, 1/fan_in)
    b1 = w[nt * F + F * K: nt * F + F * K + F]
    assert np.all(b1 == 0.0)                                   # biases 0 in the configs
