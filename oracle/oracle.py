"""ctypes binding of the double-precision CPU oracle (sn_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the benchmark's
CPU-baseline leg, never by the library's own code path.  It computes, in double precision
and in plain loops, what FlashSchNet (arXiv 2602.13140, §3.2 and §4) defines: the
neighbour list, the SchNet energy and its analytic forces, and velocity Verlet.
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "sn_oracle.c"
LIB = HERE / "libsn_oracle.so"
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]

# The build timed as the benchmark's CPU baseline: the same source and the same IEEE
# semantics (no contraction, no fast-math), optimised for the host it runs on.  Compiled on
# that host at run time, never shipped, so -march=native cannot meet a CPU it was not built for.
NATIVE_CFLAGS = ["-O3", "-march=native", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]

_lib = None


def build_native(out_dir: Path) -> Path:
    """Compile the oracle with NATIVE_CFLAGS into out_dir (for the CPU-baseline timing)."""
    out = Path(out_dir) / "libsn_oracle_native.so"
    subprocess.check_call(["gcc", *NATIVE_CFLAGS, "-o", str(out), str(SRC), "-lm"])
    return out


def set_threads(n: int) -> None:
    """OpenMP thread count of the oracle's later parallel regions (the process's libgomp)."""
    C.CDLL("libgomp.so.1").omp_set_num_threads(C.c_int(int(n)))


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if force or not LIB.exists() or LIB.stat().st_mtime < SRC.stat().st_mtime:
        tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(["gcc", *CFLAGS, "-o", str(tmp), str(SRC), "-lm"])
        os.replace(tmp, LIB)
    return LIB


def compile_variant(src_text: str, out: Path) -> Path:
    """Compile a modified copy of the oracle's source (used by the tests that plant
    mistakes in the oracle to show that its pins catch them)."""
    src = out.with_suffix(".c")
    src.write_text(src_text)
    subprocess.check_call(["gcc", *CFLAGS, "-o", str(out), str(src), "-lm"])
    return out


@contextlib.contextmanager
def using(path: Path):
    """Route every call of this module to another build of the oracle while inside."""
    global _lib
    saved = _lib
    _lib = _load(path)
    try:
        yield
    finally:
        _lib = saved


def lib():
    global _lib
    if _lib is None:
        _lib = _load(build())
    return _lib


def _load(path):
    L = C.CDLL(str(path))
    P = C.c_void_p
    i64, f32, f64 = C.c_int64, C.c_float, C.c_double
    L.sno_pair_within.argtypes = [P, P, P, f32]
    L.sno_pair_within.restype = C.c_int
    for fn in (L.sno_neighbors_brute, L.sno_neighbors_cells):
        fn.argtypes = [C.c_int, C.c_int, P, f32, P, i64, P, P, P]
        fn.restype = C.c_int
    for fn in (L.sno_energy_forces, L.sno_energy_forces_f64):
        fn.argtypes = [P, f64, f64, P, i64, C.c_int, C.c_int, P, P, P, P, P, i64, P, P, P]
        fn.restype = C.c_int
    L.sno_md_vv.argtypes = [P, f64, f64, P, i64, C.c_int, C.c_int, P, P, P, P, P,
                            f64, f64, C.c_int, P, P, P]
    L.sno_md_vv.restype = C.c_int
    L.sno_num_threads.restype = C.c_int
    L.sno_philox4x32_10.argtypes = [P, P, P]
    L.sno_philox4x32_10.restype = None
    L.sno_langevin_noise.argtypes = [C.c_uint64, C.c_int64, C.c_int64, P]
    L.sno_langevin_noise.restype = None
    L.sno_md_langevin.argtypes = [P, f64, f64, P, i64, C.c_int, C.c_int, P, P, P, P, P,
                                  f64, f64, C.c_int, f64, f64, C.c_uint64, C.c_int64, P, P]
    L.sno_md_langevin.restype = C.c_int
    return L


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _box(system) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(system.box, dtype=np.float32).reshape(3))


def num_threads() -> int:
    return lib().sno_num_threads()


def pair_within(pi, pj, box, r_cut) -> bool:
    a = np.ascontiguousarray(pi, dtype=np.float32)
    b = np.ascontiguousarray(pj, dtype=np.float32)
    bx = np.ascontiguousarray(box, dtype=np.float32)
    return bool(lib().sno_pair_within(_p(a), _p(b), _p(bx), C.c_float(r_cut)))


def neighbors(system, r_cut: float, pos: np.ndarray, method: str = "brute", cap: int | None = None):
    """CSR neighbour list (row_ptr int32 [N+1], col int32 [E]), rows by destination,
    sources ascending.  Raises OverflowError(n_needed) if cap is too small."""
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    N = system.n_atoms
    if cap is None:
        cap = max(N * 64, 64)
    row_ptr = np.zeros(N + 1, dtype=np.int32)
    col = np.zeros(max(cap, 1), dtype=np.int32)
    ne = np.zeros(1, dtype=np.int64)
    fn = lib().sno_neighbors_cells if method == "cells" else lib().sno_neighbors_brute
    box = _box(system)
    st = fn(system.n_per_replica, system.n_replicas, _p(box), C.c_float(r_cut), _p(pos),
            C.c_int64(cap), _p(row_ptr), _p(col), _p(ne))
    if st == 2:  # too small: retry with the size the oracle asked for
        return neighbors(system, r_cut, pos, method, cap=int(ne[0]) + 1)
    if st != 0:
        raise ValueError(f"oracle neighbour build failed: status {st}")
    return row_ptr, col[: int(ne[0])].copy()


def _dims(model) -> np.ndarray:
    return np.array([model.F, model.K, model.T, model.n_types], dtype=np.int32)


def energy_forces(model, weights, system, pos, types, row_ptr, col, f64_pos: bool = False):
    """Energies per replica [R], forces [N][3] and per-atom energies [N], all float64."""
    N, R = system.n_atoms, system.n_replicas
    dims = _dims(model)
    w = np.ascontiguousarray(weights, dtype=np.float32)
    types = np.ascontiguousarray(types, dtype=np.int32)
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    col = np.ascontiguousarray(col, dtype=np.int32)
    if col.size == 0:
        col = np.zeros(1, dtype=np.int32)
    energy = np.zeros(max(R, 1))
    forces = np.zeros((max(N, 1), 3))
    eps = np.zeros(max(N, 1))
    box = _box(system)
    if f64_pos:
        p = np.ascontiguousarray(pos, dtype=np.float64)
        fn = lib().sno_energy_forces_f64
    else:
        p = np.ascontiguousarray(pos, dtype=np.float32)
        fn = lib().sno_energy_forces
    st = fn(_p(dims), C.c_double(model.r_cut), C.c_double(model.gamma), _p(w), C.c_int64(w.size),
            system.n_per_replica, system.n_replicas, _p(box), _p(p), _p(types), _p(row_ptr),
            _p(col), C.c_int64(int(row_ptr[-1]) if N else 0), _p(energy), _p(forces), _p(eps))
    if st != 0:
        raise ValueError(f"oracle energy/forces failed: status {st}")
    return energy[:R], forces[:N], eps[:N]


def md_vv(model, weights, system, pos, vel, types, mass, dt, n_steps, forces=None):
    """Velocity-Verlet NVE in double.  Returns (pos, vel, forces, epot[n_steps][R],
    ekin[n_steps][R], n_edges_last).  If forces is None, F(t0) is computed first."""
    N, R = system.n_atoms, system.n_replicas
    pos = np.array(pos, dtype=np.float64, copy=True)
    vel = np.array(vel, dtype=np.float64, copy=True)
    if forces is None:
        rp, cl = neighbors(system, model.r_cut, pos.astype(np.float32),
                           "cells" if system.periodic else "brute")
        _, forces, _ = energy_forces(model, weights, system, pos, types, rp, cl, f64_pos=True)
    forces = np.array(forces, dtype=np.float64, copy=True)
    dims = _dims(model)
    w = np.ascontiguousarray(weights, dtype=np.float32)
    types = np.ascontiguousarray(types, dtype=np.int32)
    epot = np.zeros((max(n_steps, 1), R))
    ekin = np.zeros((max(n_steps, 1), R))
    ne = np.zeros(1, dtype=np.int64)
    box = _box(system)
    st = lib().sno_md_vv(_p(dims), C.c_double(model.r_cut), C.c_double(model.gamma), _p(w),
                         C.c_int64(w.size), system.n_per_replica, system.n_replicas, _p(box),
                         _p(pos), _p(vel), _p(forces), _p(types), C.c_double(mass),
                         C.c_double(dt), n_steps, _p(epot), _p(ekin), _p(ne))
    if st != 0:
        raise ValueError(f"oracle MD failed: status {st}")
    return pos, vel, forces, epot[:n_steps], ekin[:n_steps], int(ne[0])


def philox4x32_10(ctr, key):
    """Philox4x32-10 of a 4-word counter and 2-word key (uint32 words)."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().sno_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def langevin_noise(seed: int, step: int, atom: int) -> np.ndarray:
    xi = np.zeros(3)
    lib().sno_langevin_noise(C.c_uint64(seed), C.c_int64(step), C.c_int64(atom), _p(xi))
    return xi


def md_langevin(model, weights, system, pos, vel, types, mass, dt, n_steps, temperature, friction,
                seed, step0=0, forces=None):
    """BAOAB Langevin in double.  Returns (pos, vel, forces, epot[n][R], ekin[n][R])."""
    N, R = system.n_atoms, system.n_replicas
    pos = np.array(pos, dtype=np.float64, copy=True)
    vel = np.array(vel, dtype=np.float64, copy=True)
    if forces is None:
        rp, cl = neighbors(system, model.r_cut, pos.astype(np.float32),
                           "cells" if system.periodic else "brute")
        _, forces, _ = energy_forces(model, weights, system, pos, types, rp, cl, f64_pos=True)
    forces = np.array(forces, dtype=np.float64, copy=True)
    w = np.ascontiguousarray(weights, dtype=np.float32)
    types = np.ascontiguousarray(types, dtype=np.int32)
    epot = np.zeros((max(n_steps, 1), R))
    ekin = np.zeros((max(n_steps, 1), R))
    box = _box(system)
    st = lib().sno_md_langevin(_p(_dims(model)), C.c_double(model.r_cut), C.c_double(model.gamma), _p(w),
                               C.c_int64(w.size), system.n_per_replica, system.n_replicas, _p(box), _p(pos),
                               _p(vel), _p(forces), _p(types), C.c_double(mass), C.c_double(dt), n_steps,
                               C.c_double(temperature), C.c_double(friction), C.c_uint64(seed),
                               C.c_int64(step0), _p(epot), _p(ekin))
    if st != 0:
        raise ValueError(f"oracle Langevin failed: status {st}")
    return pos, vel, forces, epot[:n_steps], ekin[:n_steps]
