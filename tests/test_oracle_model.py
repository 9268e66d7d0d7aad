"""Pins of the oracle's energy and analytic forces (CPU only).

Nothing here calls the oracle to check the oracle.  The pins are:
  - a closed form of the whole model for two atoms, written out feature by feature;
  - the T = 0 special case (energy = readout of the embeddings, forces = 0);
  - central finite differences of the energy (pins the hand-written backward);
  - invariances the physics fixes: translation, rotation, permutation, replica independence,
    sum of forces = 0, and continuity of E at the cutoff when the filter biases are zero.
Mistakes these catch: swapped src/dst in the message, a transposed weight, a dropped bias,
the envelope on the wrong factor, a wrong sign or index in the backward.
"""
import math

import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth


def _ssp(x):
    return math.log(0.5 * math.exp(x) + 0.5)


def _unpack(blob, F, K, T, n_types):
    """Split the blob into named arrays following the documented layout."""
    H = F // 2
    out, p = {}, 0

    def take(name, shape):
        nonlocal p
        n = int(np.prod(shape))
        out[name] = blob[p:p + n].astype(np.float64).reshape(shape)
        p += n

    take("emb", (n_types, F))
    for t in range(T):
        take(f"W1_{t}", (F, K)); take(f"b1_{t}", (F,))
        take(f"W2_{t}", (F, F)); take(f"b2_{t}", (F,))
        take(f"U1_{t}", (F, F)); take(f"c1_{t}", (F,))
        take(f"U2_{t}", (F, F)); take(f"c2_{t}", (F,))
    take("R1", (H, F)); take("e1", (H,)); take("R2", (1, H)); take("e2", (1,))
    assert p == blob.size
    return out


def closed_form_two_atoms(blob, d, z0, z1, r_cut, gamma, F=2, K=3, swap=False):
    """E for two atoms at distance d, F = 2 features, K = 3 Gaussians, T = 1, H = 1.
    Written out component by component (no matrix routines).  swap=True plants the mistake
    of gathering the destination's own features instead of the source's."""
    P = _unpack(blob, F, K, 1, 3)
    mu = [k * r_cut / (K - 1) for k in range(K)]
    env = 0.5 * (math.cos(math.pi * d / r_cut) + 1.0)
    bt = [math.exp(-gamma * (d - mu[k]) ** 2) * env for k in range(K)]
    W1, b1, W2, b2 = P["W1_0"], P["b1_0"], P["W2_0"], P["b2_0"]
    a0 = W1[0, 0] * bt[0] + W1[0, 1] * bt[1] + W1[0, 2] * bt[2] + b1[0]
    a1 = W1[1, 0] * bt[0] + W1[1, 1] * bt[1] + W1[1, 2] * bt[2] + b1[1]
    s0, s1 = _ssp(a0), _ssp(a1)
    w0 = W2[0, 0] * s0 + W2[0, 1] * s1 + b2[0]
    w1 = W2[1, 0] * s0 + W2[1, 1] * s1 + b2[1]
    x = {0: P["emb"][z0], 1: P["emb"][z1]}
    # atom 0 receives from atom 1 and vice versa: h_i = x_j (.) w
    h = {0: (x[1][0] * w0, x[1][1] * w1), 1: (x[0][0] * w0, x[0][1] * w1)}
    if swap:
        h = {0: (x[0][0] * w0, x[0][1] * w1), 1: (x[1][0] * w0, x[1][1] * w1)}
    U1, c1, U2, c2 = P["U1_0"], P["c1_0"], P["U2_0"], P["c2_0"]
    R1, e1, R2, e2 = P["R1"], P["e1"], P["R2"], P["e2"]
    E = 0.0
    for i in (0, 1):
        p0 = U1[0, 0] * h[i][0] + U1[0, 1] * h[i][1] + c1[0]
        p1 = U1[1, 0] * h[i][0] + U1[1, 1] * h[i][1] + c1[1]
        q0, q1 = _ssp(p0), _ssp(p1)
        y0 = x[i][0] + U2[0, 0] * q0 + U2[0, 1] * q1 + c2[0]
        y1 = x[i][1] + U2[1, 0] * q0 + U2[1, 1] * q1 + c2[1]
        o = R1[0, 0] * y0 + R1[0, 1] * y1 + e1[0]
        E += R2[0, 0] * _ssp(o) + e2[0]
    return E


@pytest.mark.parametrize("d", [1.3, 2.71, 4.4])
def test_closed_form_two_atoms(oracle, d):
    r_cut, gamma = 5.0, 0.7
    model = synth.ModelCfg(F=2, K=3, T=1, n_types=3, r_cut=r_cut, gamma=gamma)
    blob = synth.weights_blob(2, 3, 1, 3, seed=77, bias_std=0.3)
    system = synth.SystemCfg(2, 1)
    u = np.array([0.6, -0.48, 0.64])
    u /= np.linalg.norm(u)
    pos = np.stack([np.zeros(3), u * d]).astype(np.float64)
    types = np.array([2, 0], np.int32)
    rp = np.array([0, 1, 2], np.int32)
    cl = np.array([1, 0], np.int32)
    E, Fr, eps = oracle.energy_forces(model, blob, system, pos, types, rp, cl, f64_pos=True)
    Ec = closed_form_two_atoms(blob, d, 2, 0, r_cut, gamma)
    assert E[0] == pytest.approx(Ec, rel=1e-13, abs=1e-13)
    # force on atom 1 = -dE/dd * u (u points from atom 0 to atom 1); dE/dd of the closed form
    # by a 4th-order central difference
    hh = 1e-4
    dEdd = (-closed_form_two_atoms(blob, d + 2 * hh, 2, 0, r_cut, gamma)
            + 8 * closed_form_two_atoms(blob, d + hh, 2, 0, r_cut, gamma)
            - 8 * closed_form_two_atoms(blob, d - hh, 2, 0, r_cut, gamma)
            + closed_form_two_atoms(blob, d - 2 * hh, 2, 0, r_cut, gamma)) / (12 * hh)
    np.testing.assert_allclose(Fr[1], -dEdd * u, rtol=1e-8, atol=1e-10)
    np.testing.assert_allclose(Fr[0], dEdd * u, rtol=1e-8, atol=1e-10)


def test_message_direction_matters(oracle):
    """The closed form separates x_src (.) w from the planted x_dst (.) w, and the oracle
    sides with x_src."""
    r_cut, gamma = 5.0, 0.7
    model = synth.ModelCfg(F=2, K=3, T=1, n_types=3, r_cut=r_cut, gamma=gamma)
    blob = synth.weights_blob(2, 3, 1, 3, seed=78, bias_std=0.3)
    system = synth.SystemCfg(2, 1)
    pos = np.array([[0, 0, 0], [2.2, 0, 0]], np.float64)
    rp = np.array([0, 1, 2], np.int32)
    cl = np.array([1, 0], np.int32)
    E, _, _ = oracle.energy_forces(model, blob, system, pos, np.array([0, 1], np.int32), rp, cl, f64_pos=True)
    right = closed_form_two_atoms(blob, 2.2, 0, 1, r_cut, gamma)
    wrong = closed_form_two_atoms(blob, 2.2, 0, 1, r_cut, gamma, swap=True)
    assert abs(right - wrong) > 1e-3 * max(1.0, abs(right))
    assert E[0] == pytest.approx(right, rel=1e-13)


def test_T0_is_readout_of_embedding(oracle):
    F, K, n_types = 8, 5, 4
    model = synth.ModelCfg(F=F, K=K, T=0, n_types=n_types, r_cut=6.0)
    blob = synth.weights_blob(F, K, 0, n_types, seed=5, bias_std=0.2)
    system = synth.SystemCfg(12, 2)
    w = synth.make_custom(model, system, seed=9)
    rp, cl = oracle.neighbors(system, 6.0, w.pos)
    E, Fr, eps = oracle.energy_forces(model, blob, system, w.pos, w.types, rp, cl)
    P = _unpack(blob, F, K, 0, n_types)
    for i in range(system.n_atoms):
        xi = P["emb"][w.types[i]]
        o = [sum(P["R1"][k, f] * xi[f] for f in range(F)) + P["e1"][k] for k in range(F // 2)]
        ref = sum(P["R2"][0, k] * _ssp(o[k]) for k in range(F // 2)) + P["e2"][0]
        assert eps[i] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    assert np.all(Fr == 0.0)
    assert E[0] == pytest.approx(eps[:12].sum(), rel=1e-13)


def _fd_setup(kind, seed):
    if kind == "chain":
        model = synth.ModelCfg(F=8, K=6, T=2, n_types=3, r_cut=7.0, gamma=1.5)
        system = synth.SystemCfg(9, 2)
        w = synth.make_custom(model, system, seed, "rw", bias_std=0.2)
    else:
        model = synth.ModelCfg(F=6, K=5, T=2, n_types=2, r_cut=3.5, gamma=2.0)
        system = synth.SystemCfg(20, 1, (8.0, 8.5, 9.0))
        w = synth.make_custom(model, system, seed, "box", bias_std=0.2)
    return model, system, w


def _far_from_cutoff(pos, system, r_cut, rp, cl, margin=2e-3):
    pos = pos.astype(np.float64)
    N = system.n_atoms
    for i in range(N):
        r0 = (i // system.n_per_replica) * system.n_per_replica
        for j in range(r0, r0 + system.n_per_replica):
            if j == i:
                continue
            d = pos[j] - pos[i]
            for a in range(3):
                if system.box[a] > 0:
                    d[a] -= system.box[a] * np.rint(d[a] / system.box[a])
            if abs(np.linalg.norm(d) - r_cut) < margin:
                return False
    return True


@pytest.mark.parametrize("kind,seed", [("chain", 101), ("chain", 102), ("box", 103), ("box", 104)])
def test_forces_match_central_differences(oracle, kind, seed):
    model, system, w = _fd_setup(kind, seed)
    pos = w.pos.astype(np.float64)
    rp, cl = oracle.neighbors(system, model.r_cut, w.pos)
    assert len(cl) > 0
    if not _far_from_cutoff(pos, system, model.r_cut, rp, cl):
        pytest.skip("a pair sits within 2e-3 A of the cutoff for this seed")
    _, Fa, _ = oracle.energy_forces(model, w.weights, system, pos, w.types, rp, cl, f64_pos=True)
    h = 1e-5
    Ffd = np.zeros_like(Fa)
    for i in range(system.n_atoms):
        for a in range(3):
            pp = pos.copy(); pp[i, a] += h
            pm = pos.copy(); pm[i, a] -= h
            Ep, _, _ = oracle.energy_forces(model, w.weights, system, pp, w.types, rp, cl, f64_pos=True)
            Em, _, _ = oracle.energy_forces(model, w.weights, system, pm, w.types, rp, cl, f64_pos=True)
            Ffd[i, a] = -(Ep.sum() - Em.sum()) / (2 * h)
    scale = np.abs(Fa).max()
    assert scale > 1e-3
    np.testing.assert_allclose(Fa, Ffd, rtol=0, atol=1e-7 * scale + 1e-9)


def _rotation(seed):
    q, _ = np.linalg.qr(np.random.default_rng(seed).standard_normal((3, 3)))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def test_invariances_open_chains(oracle):
    model = synth.ModelCfg(F=16, K=10, T=3, n_types=5, r_cut=9.0, gamma=1.0)
    system = synth.SystemCfg(24, 3)
    w = synth.make_custom(model, system, 31, "saw", bias_std=0.1)
    pos = w.pos.astype(np.float64)
    rp, cl = oracle.neighbors(system, model.r_cut, w.pos)
    E, Fr, _ = oracle.energy_forces(model, w.weights, system, pos, w.types, rp, cl, f64_pos=True)
    # Newton III: forces of each replica sum to zero
    for r in range(3):
        np.testing.assert_allclose(Fr[r * 24:(r + 1) * 24].sum(0), 0.0, atol=1e-12 * np.abs(Fr).max())
    # rotation + translation: E invariant, F rotates (same edge list)
    Rm = _rotation(3)
    pos2 = pos @ Rm.T + np.array([3.0, -7.0, 11.0])
    E2, F2, _ = oracle.energy_forces(model, w.weights, system, pos2, w.types, rp, cl, f64_pos=True)
    np.testing.assert_allclose(E2, E, rtol=1e-12)
    np.testing.assert_allclose(F2, Fr @ Rm.T, rtol=0, atol=1e-11 * np.abs(Fr).max())
    # permutation within each replica: relabel atoms, rebuild the list, E same, F permuted
    rng = np.random.default_rng(4)
    perm = np.concatenate([r * 24 + rng.permutation(24) for r in range(3)])
    pos3 = pos[perm]
    rp3, cl3 = oracle.neighbors(system, model.r_cut, pos3.astype(np.float32))
    E3, F3, _ = oracle.energy_forces(model, w.weights, system, pos3, w.types[perm], rp3, cl3, f64_pos=True)
    np.testing.assert_allclose(E3, E, rtol=1e-12)
    np.testing.assert_allclose(F3, Fr[perm], rtol=0, atol=1e-12 * np.abs(Fr).max())
    # replica independence: each replica alone gives the same energy and forces
    for r in range(3):
        s1 = synth.SystemCfg(24, 1)
        p1 = pos[r * 24:(r + 1) * 24]
        rp1, cl1 = oracle.neighbors(s1, model.r_cut, p1.astype(np.float32))
        E1, F1, _ = oracle.energy_forces(model, w.weights, s1, p1, w.types[r * 24:(r + 1) * 24], rp1, cl1, f64_pos=True)
        assert E1[0] == pytest.approx(E[r], rel=1e-13)
        np.testing.assert_allclose(F1, Fr[r * 24:(r + 1) * 24], rtol=0, atol=1e-14 * np.abs(Fr).max() + 1e-15)


def test_periodic_translation_and_image_invariance(oracle):
    model = synth.ModelCfg(F=8, K=6, T=2, n_types=3, r_cut=4.0, gamma=1.0)
    system = synth.SystemCfg(60, 1, (10.0, 11.0, 12.0))
    w = synth.make_custom(model, system, 41, "box", bias_std=0.1)
    pos = w.pos.astype(np.float64)
    rp, cl = oracle.neighbors(system, model.r_cut, w.pos)
    E, Fr, _ = oracle.energy_forces(model, w.weights, system, pos, w.types, rp, cl, f64_pos=True)
    np.testing.assert_allclose(Fr.sum(0), 0.0, atol=1e-12 * np.abs(Fr).max())
    # shifting single atoms by whole box vectors changes nothing
    pos2 = pos.copy()
    pos2[::3] += np.array([10.0, -11.0, 24.0])
    E2, F2, _ = oracle.energy_forces(model, w.weights, system, pos2, w.types, rp, cl, f64_pos=True)
    np.testing.assert_allclose(E2, E, rtol=1e-12)
    np.testing.assert_allclose(F2, Fr, rtol=0, atol=1e-11 * np.abs(Fr).max())


def test_energy_continuous_at_cutoff(oracle):
    """With zero filter biases the filter vanishes with the envelope at r_cut, so the
    energy of a pair approaches that of two isolated atoms, with zero slope."""
    r_cut = 5.0
    model = synth.ModelCfg(F=4, K=5, T=2, n_types=2, r_cut=r_cut, gamma=1.0)
    blob = synth.weights_blob(4, 5, 2, 2, seed=8, bias_std=0.0)
    system = synth.SystemCfg(2, 1)
    types = np.array([0, 1], np.int32)
    edge = (np.array([0, 1, 2], np.int32), np.array([1, 0], np.int32))
    none = (np.array([0, 0, 0], np.int32), np.zeros(0, np.int32))

    def energy(d, graph):
        pos = np.array([[0, 0, 0], [d, 0, 0]], np.float64)
        return oracle.energy_forces(model, blob, system, pos, types, *graph, f64_pos=True)

    E_iso = energy(6.0, none)[0][0]
    for eps_d in (1e-2, 1e-3):
        E_near, F_near, _ = energy(r_cut - eps_d, edge)
        assert abs(E_near[0] - E_iso) < 50 * eps_d ** 2 * max(1.0, abs(E_iso))
        assert np.abs(F_near).max() < 50 * eps_d


def test_zero_filter_gives_position_independent_energy(oracle):
    F, K, T, nt = 8, 4, 2, 3
    model = synth.ModelCfg(F=F, K=K, T=T, n_types=nt, r_cut=6.0)
    blob = synth.weights_blob(F, K, T, nt, seed=12, bias_std=0.3)
    # zero the second filter layer (W2, b2) in every block
    H = F // 2
    p = nt * F
    for t in range(T):
        p += F * K + F
        blob[p:p + F * F + F] = 0.0
        p += F * F + F
        p += 2 * (F * F + F)
    system = synth.SystemCfg(10, 1)
    w = synth.make_custom(model, system, 3)
    rp, cl = oracle.neighbors(system, 6.0, w.pos)
    assert len(cl) > 0
    E, Fr, _ = oracle.energy_forces(model, blob, system, w.pos, w.types, rp, cl)
    assert np.all(Fr == 0.0)
    iso = oracle.energy_forces(model, blob, system, w.pos * 100, w.types, np.zeros(11, np.int32), np.zeros(0, np.int32))[0]
    assert E[0] == pytest.approx(iso[0], rel=1e-13)
