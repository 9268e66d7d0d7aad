"""Seeded synthetic inputs: bead chains, periodic boxes, bead types, weight blobs, velocities.

This module is shared by the CPU oracle's tests and by the CUDA path (tests, smoke, bench).
It holds none of the method's arithmetic: it only draws random numbers and lays them out.

Workloads (FlashSchNet, arXiv 2602.13140, §5.1 "Experimental setting": 64 replicas of a
coarse-grained protein of 269 beads; the proteins themselves are not available, so seeded
random-walk chains of the same size stand in for them):

  cfg1  tiny chain: 1 x 32 beads, 3D random walk, 3.8 A bonds, 4 types, r_c 10 A, open;
        F 64, K 32, T 2
  cfg2  64 x 269 self-avoiding random-walk chains, 20 types, r_c 12 A, open; F 128, K 50, T 3
  cfg3  cfg2 run as NVE velocity-Verlet MD: dt 2 fs, 12 amu beads, 300 K, 1000 steps
  cfg4  4096 atoms uniform in a periodic 40.6 A cube, 8 species, r_c 5 A; F 128, K 50, T 3
  cfg5  65,536 atoms uniform in a periodic 102.3 A cube, r_c 5 A; F 128, K 50, T 3; 100 MD steps

Weight blob (float32, one flat array), in this order; every Linear is W[out][in] row-major
followed by its bias[out] (y = W x + b):
  Emb[n_types][F]
  per interaction block t = 0..T-1:
      W1[F][K], b1[F], W2[F][F], b2[F]      (filter network K -> F -> F)
      U1[F][F], c1[F], U2[F][F], c2[F]      (update network F -> F -> F, residual)
  R1[F/2][F], e1[F/2], R2[1][F/2], e2[1]    (readout F -> F/2 -> 1)
Linear weights ~ N(0, 1/fan_in); biases 0 unless bias_std > 0; Emb ~ N(0, 1).
"""
from __future__ import annotations

import dataclasses
import numpy as np

BOND = 3.8            # A, bead-bead bond length of the chains
KB = 0.0019872041     # kcal/mol/K
KAPPA = 4.184e-4      # A^2 fs^-2 per (kcal/mol)/amu


@dataclasses.dataclass(frozen=True)
class ModelCfg:
    F: int
    K: int
    T: int
    n_types: int
    r_cut: float
    gamma: float = 10.0


@dataclasses.dataclass(frozen=True)
class SystemCfg:
    n_per_replica: int
    n_replicas: int
    box: tuple = (0.0, 0.0, 0.0)   # all zero = open boundaries

    @property
    def n_atoms(self) -> int:
        return self.n_per_replica * self.n_replicas

    @property
    def periodic(self) -> bool:
        return any(b > 0 for b in self.box)


@dataclasses.dataclass
class Workload:
    name: str
    model: ModelCfg
    system: SystemCfg
    pos: np.ndarray        # float32 [N][3]
    types: np.ndarray      # int32 [N]
    weights: np.ndarray    # float32 flat blob
    md: dict | None = None


def n_weights(F: int, K: int, T: int, n_types: int) -> int:
    H = F // 2
    per_block = F * K + F + F * F + F + F * F + F + F * F + F
    return n_types * F + T * per_block + H * F + H + H + 1


def weights_blob(F: int, K: int, T: int, n_types: int, seed: int,
                 bias_std: float = 0.0) -> np.ndarray:
    """Draw the weight blob in the documented order with numpy default_rng(seed)."""
    rng = np.random.default_rng(seed)
    parts = [rng.standard_normal((n_types, F))]

    def linear(n_out, n_in):
        w = rng.standard_normal((n_out, n_in)) / np.sqrt(n_in)
        b = rng.standard_normal(n_out) * bias_std if bias_std > 0 else np.zeros(n_out)
        parts.append(w)
        parts.append(b)

    for _ in range(T):
        linear(F, K)
        linear(F, F)
        linear(F, F)
        linear(F, F)
    linear(F // 2, F)
    linear(1, F // 2)
    blob = np.concatenate([p.ravel() for p in parts]).astype(np.float32)
    assert blob.size == n_weights(F, K, T, n_types)
    return blob


def _unit_vectors(rng, n):
    v = rng.standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def random_walk(n: int, rng, bond: float = BOND) -> np.ndarray:
    """Free 3D random walk from the origin, fixed bond length, uniform directions."""
    steps = _unit_vectors(rng, n - 1) * bond
    pos = np.zeros((n, 3))
    pos[1:] = np.cumsum(steps, axis=0)
    return pos


def self_avoiding_walk(n: int, rng, bond: float = BOND, max_tries: int = 1000) -> np.ndarray:
    """Random walk that rejects a step landing closer than one bond to any earlier,
    non-bonded bead; retries a step up to max_tries times, restarts the chain on failure."""
    while True:
        pos = np.zeros((n, 3))
        ok = True
        for i in range(1, n):
            placed = False
            for _ in range(max_tries):
                cand = pos[i - 1] + _unit_vectors(rng, 1)[0] * bond
                if i >= 2:
                    d2 = np.sum((pos[: i - 1] - cand) ** 2, axis=1)
                    if np.any(d2 < bond * bond):
                        continue
                pos[i] = cand
                placed = True
                break
            if not placed:
                ok = False
                break
        if ok:
            return pos


def uniform_box(n: int, box, rng) -> np.ndarray:
    """Uniform positions in [0, L_x) x [0, L_y) x [0, L_z), float32."""
    return (rng.random((n, 3)) * np.asarray(box, dtype=np.float64)).astype(np.float32)


def chains(n_per: int, n_rep: int, seed: int, saw: bool) -> np.ndarray:
    rng = np.random.default_rng(seed)
    walk = self_avoiding_walk if saw else random_walk
    return np.concatenate([walk(n_per, rng) for _ in range(n_rep)]).astype(np.float32)


def bead_types(n: int, n_types: int, seed: int) -> np.ndarray:
    return np.random.default_rng(seed).integers(0, n_types, size=n).astype(np.int32)


def maxwell_boltzmann(n_per: int, n_rep: int, mass: float, temp: float, seed: int) -> np.ndarray:
    """Velocities (A/fs) drawn per component from N(0, kB*T*kappa/m), then the centre-of-mass
    velocity of each replica is removed (equal masses). float32 [N][3]."""
    rng = np.random.default_rng(seed)
    sigma = np.sqrt(KB * temp * KAPPA / mass)
    v = rng.standard_normal((n_rep, n_per, 3)) * sigma
    v -= v.mean(axis=1, keepdims=True)
    return v.reshape(-1, 3).astype(np.float32)


CONFIGS = {
    1: dict(name="tiny chain 1x32, r_c 10, F64 K32 T2",
            model=ModelCfg(F=64, K=32, T=2, n_types=4, r_cut=10.0),
            system=SystemCfg(32, 1), kind="rw"),
    2: dict(name="64x269 SAW chains, r_c 12, F128 K50 T3",
            model=ModelCfg(F=128, K=50, T=3, n_types=20, r_cut=12.0),
            system=SystemCfg(269, 64), kind="saw"),
    3: dict(name="64x269 SAW chains NVE MD, dt 2 fs, 1000 steps",
            model=ModelCfg(F=128, K=50, T=3, n_types=20, r_cut=12.0),
            system=SystemCfg(269, 64), kind="saw",
            md=dict(dt=2.0, mass=12.0, temp=300.0, steps=1000)),
    4: dict(name="4096 atoms periodic 40.6 A cube, r_c 5, F128 K50 T3",
            model=ModelCfg(F=128, K=50, T=3, n_types=8, r_cut=5.0),
            system=SystemCfg(4096, 1, (40.6, 40.6, 40.6)), kind="box"),
    5: dict(name="65536 atoms periodic 102.3 A cube, r_c 5, F128 K50 T3",
            model=ModelCfg(F=128, K=50, T=3, n_types=8, r_cut=5.0),
            system=SystemCfg(65536, 1, (102.3, 102.3, 102.3)), kind="box",
            md=dict(dt=2.0, mass=12.0, temp=300.0, steps=100)),
}


def make_workload(cfg: int, bias_std: float = 0.0) -> Workload:
    """The seeded workload of configuration `cfg` (seeds: positions 1000+cfg, types 2000+cfg,
    weights 3000+cfg, velocities 4000+cfg)."""
    c = CONFIGS[cfg]
    m, s = c["model"], c["system"]
    if c["kind"] == "box":
        pos = uniform_box(s.n_atoms, s.box, np.random.default_rng(1000 + cfg))
    else:
        pos = chains(s.n_per_replica, s.n_replicas, 1000 + cfg, saw=(c["kind"] == "saw"))
    types = bead_types(s.n_atoms, m.n_types, 2000 + cfg)
    w = weights_blob(m.F, m.K, m.T, m.n_types, 3000 + cfg, bias_std=bias_std)
    return Workload(c["name"], m, s, pos, types, w, c.get("md"))


def make_custom(model: ModelCfg, system: SystemCfg, seed: int, kind: str = "rw",
                bias_std: float = 0.0) -> Workload:
    """Seeded workload of any size (tests: ragged sizes, tiny systems, other boxes)."""
    if kind == "box":
        pos = uniform_box(system.n_atoms, system.box, np.random.default_rng(seed))
    else:
        pos = chains(system.n_per_replica, system.n_replicas, seed, saw=(kind == "saw"))
    types = bead_types(system.n_atoms, model.n_types, seed + 1)
    w = weights_blob(model.F, model.K, model.T, model.n_types, seed + 2, bias_std=bias_std)
    return Workload(f"custom-{seed}", model, system, pos, types, w, None)
