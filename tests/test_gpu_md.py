"""Velocity Verlet on the GPU (sn_md_step) vs the oracle's double-precision integrator."""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _start(oracle, w, dev):
    from schnet_gnn_molecular_cell_b200 import Context
    s, m = w.system, w.model
    v0 = synth.maxwell_boltzmann(s.n_per_replica, s.n_replicas, 12.0, 300.0, seed=4003)
    ctx = Context(m, w.weights)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    e0, f0 = ctx.energy_forces(s, pos, types, rp, cl)
    return ctx, v0, pos, vel, types, f0.clone()


@pytest.mark.parametrize("cfg,steps", [(1, 10), (2, 3), (4, 3)])
def test_md_matches_oracle(oracle, dev, cfg, steps):
    """Two checks.  (1) The trajectory follows the oracle's double-precision one: positions
    are stored in fp32 (precision contract), each drift rounds r + dt v to within 2^-24 |r|,
    so allow 1e-6 |r| + 1e-5 A; velocities and kinetic energy to 1e-4.  (2) Energy and
    forces at the GPU's own final positions equal the oracle's at those positions, within
    the fp32 energy/force tolerance (forces at the oracle's slightly different positions
    differ by the Hessian times that rounding, which is not a property of the kernels)."""
    from tests.test_gpu_parity import assert_close
    w = synth.make_workload(cfg)
    s = w.system
    ctx, v0, pos, vel, types, forces = _start(oracle, w, dev)
    energy = torch.empty(s.n_replicas, device=dev)
    kin = torch.empty(s.n_replicas, device=dev)
    ctx.md_step(s, pos, vel, forces, types, 12.0, 2.0, steps, energy, kin)
    ctx.sync()
    p_o, v_o, f_o, epot, ekin, _ = oracle.md_vv(w.model, w.weights, s, w.pos, v0, w.types, 12.0, 2.0, steps)
    p_g = pos.cpu().numpy()
    np.testing.assert_allclose(p_g, p_o, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(vel.cpu().numpy(), v_o, rtol=1e-4, atol=1e-7)
    np.testing.assert_allclose(kin.cpu().numpy(), ekin[-1], rtol=1e-4, atol=1e-5)
    rp, cl = oracle.neighbors(s, w.model.r_cut, p_g, "cells" if s.periodic else "brute")
    E_o, F_o, _ = oracle.energy_forces(w.model, w.weights, s, p_g, w.types, rp, cl)
    assert_close(energy.cpu().numpy(), E_o, "energy at final positions")
    assert_close(forces.cpu().numpy(), F_o, "forces at final positions")
    assert ctx.md_edges() == len(cl)


def test_md_host_variant_equals_device(oracle, dev):
    w = synth.make_workload(1)
    s = w.system
    ctx, v0, pos, vel, types, forces = _start(oracle, w, dev)
    p_h, v_h, f_h = w.pos.copy(), v0.copy(), forces.cpu().numpy().copy()
    e_h = np.zeros(1, np.float32)
    k_h = np.zeros(1, np.float32)
    energy = torch.empty(1, device=dev)
    kin = torch.empty(1, device=dev)
    ctx.md_step(s, pos, vel, forces, types, 12.0, 2.0, 5, energy, kin)
    ctx.sync()
    ctx.md_step_host(s, p_h, v_h, f_h, w.types.copy(), 12.0, 2.0, 5, e_h, k_h)
    assert np.array_equal(p_h, pos.cpu().numpy())
    assert np.array_equal(v_h, vel.cpu().numpy())
    assert np.array_equal(f_h, forces.cpu().numpy())
    assert np.array_equal(e_h, energy.cpu().numpy()) and np.array_equal(k_h, kin.cpu().numpy())


def test_md_capacity_overflow_is_latched(dev):
    from schnet_gnn_molecular_cell_b200 import SNError, Status
    w = synth.make_workload(1)
    s = w.system
    from schnet_gnn_molecular_cell_b200 import Context
    ctx = Context(w.model, w.weights)
    ctx.reserve(s, 16)                       # far too small for ~576 edges
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.zeros_like(pos)
    forces = torch.zeros_like(pos)
    types = torch.from_numpy(w.types).to(dev)
    e = torch.empty(1, device=dev)
    k = torch.empty(1, device=dev)
    ctx.md_step(s, pos, vel, forces, types, 12.0, 2.0, 2, e, k)
    with pytest.raises(SNError) as ei:
        ctx.sync()
    assert ei.value.status == Status.CAPACITY
    ctx.reserve(s, 4096)
    ctx.md_step(s, pos, vel, forces, types, 12.0, 2.0, 1, e, k)
    ctx.sync()


def _zero_filter_model(n_per, n_rep, seed=9):
    """A model whose filter output is zero, so forces vanish identically."""
    F, K, T, nt = 128, 50, 1, 2
    model = synth.ModelCfg(F=F, K=K, T=T, n_types=nt, r_cut=5.0)
    blob = synth.weights_blob(F, K, T, nt, seed=3, bias_std=0.1)
    p = nt * F + F * K + F
    blob[p:p + F * F + F] = 0.0
    w = synth.make_custom(model, synth.SystemCfg(n_per, n_rep), seed, "rw")
    return model, blob, w


@pytest.mark.parametrize("precision", [0, 1, 2])
def test_langevin_o_step_uses_the_oracle_noise(oracle, dev, precision):
    from schnet_gnn_molecular_cell_b200 import Context
    model, blob, w = _zero_filter_model(64, 2)
    s = w.system
    ctx = Context(model, blob, precision=precision)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    v0 = np.full((128, 3), 0.02, np.float32)
    vel = torch.from_numpy(v0.copy()).to(dev)
    forces = torch.zeros_like(pos)
    types = torch.from_numpy(w.types).to(dev)
    e = torch.empty(2, device=dev)
    k = torch.empty(2, device=dev)
    mass, dt, temp, fr, seed, step0 = 12.0, 4.0, 300.0, 0.01, 12345, 77
    ctx.md_langevin(s, pos, vel, forces, types, mass, dt, 1, temp, fr, seed, step0, e, k)
    ctx.sync()
    a = np.exp(-fr * dt)
    b = np.sqrt((1 - a * a) * synth.KB * temp * synth.KAPPA / mass)
    xi = np.array([oracle.langevin_noise(seed, step0, i) for i in range(128)])
    v1 = a * v0 + b * xi
    np.testing.assert_allclose(vel.cpu().numpy(), v1, rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(pos.cpu().numpy(), w.pos + 0.5 * dt * (v0 + v1), rtol=1e-6, atol=1e-6)
    assert np.all(forces.cpu().numpy() == 0.0)


def test_langevin_matches_oracle(oracle, dev):
    from tests.test_gpu_parity import assert_close
    from schnet_gnn_molecular_cell_b200 import Context
    w = synth.make_workload(1)
    s = w.system
    v0 = synth.maxwell_boltzmann(32, 1, 12.0, 300.0, seed=4001)
    ctx = Context(w.model, w.weights)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    _, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    e = torch.empty(1, device=dev)
    k = torch.empty(1, device=dev)
    ctx.md_langevin(s, pos, vel, forces, types, 12.0, 4.0, 10, 300.0, 0.001, 99, 0, e, k)
    ctx.sync()
    p_o, v_o, f_o, epot, ekin = oracle.md_langevin(w.model, w.weights, s, w.pos, v0, w.types, 12.0, 4.0, 10,
                                                   300.0, 0.001, seed=99)
    p_g = pos.cpu().numpy()
    np.testing.assert_allclose(p_g, p_o, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(vel.cpu().numpy(), v_o, rtol=1e-4, atol=1e-7)
    rp, cl = oracle.neighbors(s, w.model.r_cut, p_g)
    E_o, F_o, _ = oracle.energy_forces(w.model, w.weights, s, p_g, w.types, rp, cl)
    assert_close(e.cpu().numpy(), E_o, "energy at final positions")
    assert_close(forces.cpu().numpy(), F_o, "forces at final positions")


def test_langevin_thermalises(dev):
    from schnet_gnn_molecular_cell_b200 import Context
    model, blob, w = _zero_filter_model(64, 4)
    s = w.system
    ctx = Context(model, blob, precision=1)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.full((256, 3), 0.02, device=dev)
    forces = torch.zeros_like(pos)
    types = torch.from_numpy(w.types).to(dev)
    e = torch.empty(4, device=dev)
    k = torch.empty(4, device=dev)
    ke = []
    for step in range(400):
        ctx.md_langevin(s, pos, vel, forces, types, 12.0, 4.0, 1, 300.0, 0.01, 5, step, e, k)
        if step >= 200:
            ke.append(k.cpu().numpy().copy())
    ctx.sync()
    ratio = np.mean(ke) / (1.5 * 64 * synth.KB * 300.0)
    assert abs(ratio - 1.0) < 0.05, ratio


# ------------------------------------------------------------------ tensor-core precisions
_ORACLE_TRAJ = {}


def _oracle_traj(oracle, cfg, integrator, steps):
    """The oracle's double-precision trajectory from the seeded start (cached: both tensor
    modes compare against the same one)."""
    key = (cfg, integrator, steps)
    if key not in _ORACLE_TRAJ:
        w = synth.make_workload(cfg)
        s = w.system
        v0 = synth.maxwell_boltzmann(s.n_per_replica, s.n_replicas, 12.0, 300.0, seed=4000 + cfg)
        if integrator == "vv":
            p, v, f, epot, ekin, _ = oracle.md_vv(w.model, w.weights, s, w.pos, v0, w.types, 12.0, 2.0, steps)
        else:
            p, v, f, epot, ekin = oracle.md_langevin(w.model, w.weights, s, w.pos, v0, w.types, 12.0, 4.0, steps,
                                                     300.0, 0.01, seed=77)
        _ORACLE_TRAJ[key] = (w, v0, p, v, f, ekin[-1])
    return _ORACLE_TRAJ[key]


@pytest.mark.parametrize("integrator", ["vv", "langevin"])
@pytest.mark.parametrize("precision", [1, 2], ids=["fp16", "tc32"])
@pytest.mark.parametrize("cfg", [2, 4])
def test_md_tensor_modes_match_oracle(oracle, dev, cfg, precision, integrator):
    """The benchmarked MD step in the tensor-core precisions against the oracle's trajectory
    (velocity Verlet at 2 fs as the benchmark runs it; BAOAB Langevin at 4 fs with the
    oracle's noise).  Trajectory: the deviation allowed on top of fp32 storage (as in
    test_md_matches_oracle) is what the mode's force tolerance can cause over the run,
    |dv| <= n dt kappa/m tol(F) and |dx| <= n^2 dt^2 kappa/m tol(F), tol(F) the mode's
    per-component force bound (5e-3 |F| + 5e-3 RMS(F) for fp16; the fp32 bound for tc32).
    Then energy and forces at the GPU's own final positions against the oracle at those
    positions, at the mode's tolerance."""
    from schnet_gnn_molecular_cell_b200 import Context
    from tests.test_gpu_parity import assert_close
    from tests.test_gpu_tensor import assert_close16
    steps = 3
    w, v0, p_o, v_o, f_o, ekin_o = _oracle_traj(oracle, cfg, integrator, steps)
    s = w.system
    ctx = Context(w.model, w.weights, precision=precision)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    _, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    energy = torch.empty(s.n_replicas, device=dev)
    kin = torch.empty(s.n_replicas, device=dev)
    if integrator == "vv":
        dt = 2.0
        ctx.md_step(s, pos, vel, forces, types, 12.0, dt, steps, energy, kin)
    else:
        dt = 4.0
        ctx.md_langevin(s, pos, vel, forces, types, 12.0, dt, steps, 300.0, 0.01, 77, 0, energy, kin)
    ctx.sync()
    if precision == 1:
        f_tol = 5e-3 * np.abs(f_o) + 5e-3 * np.sqrt(np.mean(f_o ** 2))
    else:
        f_tol = 1e-5 * max(1.0, np.sqrt(np.mean(f_o ** 2))) + 1e-4 * np.abs(f_o)
    acc = synth.KAPPA / 12.0 * 2.0 * f_tol           # x2: the forces change along the run
    p_g, v_g = pos.cpu().numpy().astype(np.float64), vel.cpu().numpy().astype(np.float64)
    dx_bound = 1e-6 * np.abs(p_o) + 1e-5 + (steps * dt) ** 2 * acc
    dv_bound = 1e-4 * np.abs(v_o) + 1e-7 + steps * dt * acc
    assert np.all(np.abs(p_g - p_o) <= dx_bound), float((np.abs(p_g - p_o) / dx_bound).max())
    assert np.all(np.abs(v_g - v_o) <= dv_bound), float((np.abs(v_g - v_o) / dv_bound).max())
    np.testing.assert_allclose(kin.cpu().numpy(), ekin_o, rtol=1e-3 if precision == 1 else 1e-4)
    pg32 = pos.cpu().numpy()
    rp, cl = oracle.neighbors(s, w.model.r_cut, pg32, "cells" if s.periodic else "brute")
    E_o, F_o, _ = oracle.energy_forces(w.model, w.weights, s, pg32, w.types, rp, cl)
    check = assert_close16 if precision == 1 else assert_close
    check(energy.cpu().numpy(), E_o, f"energy at final positions ({integrator})")
    check(forces.cpu().numpy(), F_o, f"forces at final positions ({integrator})")
    assert ctx.md_edges() == len(cl)


@pytest.mark.parametrize("precision,factor", [(2, 1.25), (1, 10.0)], ids=["tc32", "fp16"])
def test_nve_drift_matches_oracle(oracle, dev, precision, factor):
    """cfg3 (the chains as NVE velocity Verlet at 2 fs, 12 amu): the total-energy drift of
    replicas 0-3 over 100 GPU steps, max_t |E(t) - E(0)| / (n k_B T), against the oracle's
    double-precision drift from the same start.  At 2 fs the drift is the integrator's, so
    the fp32-accurate mode must reproduce the oracle's within 25 %; fp16 operands add energy
    noise of their own (about 4x the oracle's drift at this step), bounded at 10x."""
    from schnet_gnn_molecular_cell_b200 import Context
    steps, n_rep, mass, dt = 100, 4, 12.0, 2.0
    w = synth.make_workload(2)
    s, m = w.system, w.model
    n = s.n_per_replica
    v0 = synth.maxwell_boltzmann(n, s.n_replicas, mass, 300.0, seed=4002)
    kin0 = lambda v, r: 0.5 * mass / synth.KAPPA * (v.astype(np.float64).reshape(r, n, 3) ** 2).sum(axis=(1, 2))  # noqa: E731
    key = ("drift", steps, n_rep)
    if key not in _ORACLE_TRAJ:
        so = synth.SystemCfg(n, n_rep, s.box)
        po, vo, ty = w.pos[: n * n_rep], v0[: n * n_rep], w.types[: n * n_rep]
        _, _, _, epot, ekin, _ = oracle.md_vv(m, w.weights, so, po, vo, ty, mass, dt, steps)
        rp, cl = oracle.neighbors(so, m.r_cut, po)
        e0, _, _ = oracle.energy_forces(m, w.weights, so, po, ty, rp, cl)
        _ORACLE_TRAJ[key] = np.vstack([e0 + kin0(vo, n_rep), epot + ekin])
    et_o = _ORACLE_TRAJ[key]
    ctx = Context(m, w.weights, precision=precision)
    pos = torch.from_numpy(w.pos.copy()).to(dev)
    vel = torch.from_numpy(v0.copy()).to(dev)
    types = torch.from_numpy(w.types).to(dev)
    rp, cl = ctx.neighbors(s, pos)
    e0, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    hist = torch.empty((steps, 2, s.n_replicas), device=dev)
    for k in range(steps):
        ctx.md_step(s, pos, vel, forces, types, mass, dt, 1, hist[k, 0], hist[k, 1])
    ctx.sync()
    h = hist.double().cpu().numpy()
    et_g = np.vstack([e0.double().cpu().numpy() + kin0(v0, s.n_replicas), h[:, 0] + h[:, 1]])[:, :n_rep]
    kT = synth.KB * 300.0
    d_o = np.abs(et_o - et_o[:1]).max(axis=0) / (n * kT)
    d_g = np.abs(et_g - et_g[:1]).max(axis=0) / (n * kT)
    assert np.all(d_g < 1e-3), d_g
    assert np.all(d_g <= factor * d_o + 1e-7), (d_g.tolist(), d_o.tolist())
