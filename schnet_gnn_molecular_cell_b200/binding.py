"""Thin ctypes binding of libsnflash.so (the C ABI in include/sn.h).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  Torch provides device memory and the current CUDA stream.  There is no fallback:
if the compiled library is missing, loading fails with an error.
"""
from __future__ import annotations

import ctypes as C
import enum
from pathlib import Path

import numpy as np

LIB_PATH = Path(__file__).resolve().parent / "libsnflash.so"

# network arithmetic (sn_config.precision; see include/sn.h)
PREC_FP32 = 0      # CUDA-core fp32
PREC_FP16 = 1      # fp16 operands on the tensor cores, fp32 accumulation (weights cast as they are)
PREC_TC32 = 2      # fp32-accurate tensor-core split (hi + lo fp16 terms)
PREC_FP16_CH = 3   # fp16 operands with one scale per output channel of every weight matrix


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    CAPACITY = 2
    NONFINITE = 3
    DEGENERATE = 4
    CUDA = 5
    UNSUPPORTED = 6
    NOMEM = 7
    TIMEOUT = 8


class SNError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = Status(status)
        super().__init__(f"{self.status.name}: {message}")


class Config(C.Structure):
    _fields_ = [("F", C.c_int32), ("K", C.c_int32), ("T", C.c_int32), ("n_types", C.c_int32),
                ("r_cut", C.c_float), ("gamma", C.c_float), ("precision", C.c_int32)]


class System(C.Structure):
    _fields_ = [("n_per_replica", C.c_int32), ("n_replicas", C.c_int32), ("box", C.c_float * 3)]


class TraceEntry(C.Structure):
    _fields_ = [("name", C.c_char_p), ("launches", C.c_int64), ("total_ms", C.c_double)]


EXPORTS = ["sn_create", "sn_destroy", "sn_set_stream", "sn_reserve", "sn_build_neighbors",
           "sn_energy_forces", "sn_md_step", "sn_md_langevin", "sn_md_step_host", "sn_sync", "sn_md_edges",
           "sn_trace_enable", "sn_trace_read", "sn_build_neighbors_noalloc", "sn_last_error",
           "sn_version", "sn_set_wait_limit"]

_lib = None


def load():
    """Load libsnflash.so (built in-tree by build.py); raise if it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m schnet_gnn_molecular_cell_b200.build`")
    L = C.CDLL(str(LIB_PATH))
    P, i32, i64, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_float
    L.sn_create.argtypes = [C.POINTER(Config), P, i64, P, C.POINTER(P)]
    L.sn_destroy.argtypes = [P]
    L.sn_set_stream.argtypes = [P, P]
    L.sn_reserve.argtypes = [P, C.POINTER(System), i64]
    L.sn_build_neighbors.argtypes = [P, C.POINTER(System), P, P, P, i64, C.POINTER(i64)]
    L.sn_energy_forces.argtypes = [P, C.POINTER(System), P, P, P, P, i64, P, P]
    L.sn_md_step.argtypes = [P, C.POINTER(System), P, P, P, P, f32, f32, i32, P, P]
    L.sn_md_step_host.argtypes = [P, C.POINTER(System), P, P, P, P, f32, f32, i32, P, P]
    L.sn_md_langevin.argtypes = [P, C.POINTER(System), P, P, P, P, f32, f32, i32, f32, f32, C.c_uint64, i64, P, P]
    L.sn_md_langevin.restype = C.c_int
    L.sn_sync.argtypes = [P]
    L.sn_set_wait_limit.argtypes = [P, i64]
    L.sn_md_edges.argtypes = [P]
    L.sn_md_edges.restype = i64
    L.sn_trace_enable.argtypes = [P, i32]
    L.sn_trace_enable.restype = C.c_int
    L.sn_trace_read.argtypes = [P, C.POINTER(TraceEntry), i32]
    L.sn_trace_read.restype = i32
    L.sn_build_neighbors_noalloc.argtypes = [C.POINTER(System), f32, P, P, P, i64, C.POINTER(i64), P]
    L.sn_build_neighbors_noalloc.restype = C.c_int
    L.sn_last_error.argtypes = [P]
    L.sn_last_error.restype = C.c_char_p
    L.sn_version.restype = C.c_char_p
    for name in ("sn_create", "sn_destroy", "sn_set_stream", "sn_reserve", "sn_build_neighbors",
                 "sn_energy_forces", "sn_md_step", "sn_md_step_host", "sn_sync", "sn_set_wait_limit"):
        getattr(L, name).restype = C.c_int
    _lib = L
    return L


def system_struct(system) -> System:
    s = System()
    s.n_per_replica = int(system.n_per_replica)
    s.n_replicas = int(system.n_replicas)
    for a in range(3):
        s.box[a] = float(system.box[a])
    return s


def _ptr(t) -> int | None:
    """Raw address of a torch tensor or numpy array (None for None / empty)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data if t.size else None
    return t.data_ptr() if t.numel() else None


def _dev_check(t, dtype, name, min_numel: int = 0):
    """A contiguous tensor of `dtype` on the current CUDA device (the device whose stream and
    buffers the library uses) with at least min_numel elements; else TypeError / SNError
    (INVALID_ARG) before anything is handed to the library."""
    import torch
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous CUDA tensor of {dtype}")
    if t.device.index != torch.cuda.current_device():
        raise SNError(Status.INVALID_ARG, f"{name} is on {t.device}, the current device is "
                                          f"cuda:{torch.cuda.current_device()}")
    if t.numel() < min_numel:
        raise SNError(Status.INVALID_ARG, f"{name} has {t.numel()} elements, needs at least {min_numel}")


def _check_md_arrays(system, pos, vel, forces, types, energy, kinetic):
    import torch
    N, R = system.n_per_replica * system.n_replicas, system.n_replicas
    for t, dtp, n, k in ((pos, torch.float32, "pos", 3 * N), (vel, torch.float32, "vel", 3 * N),
                         (forces, torch.float32, "forces", 3 * N), (types, torch.int32, "types", N),
                         (energy, torch.float32, "energy", R), (kinetic, torch.float32, "kinetic", R)):
        _dev_check(t, dtp, n, k)


class Context:
    """One model (weights, workspace, stream) on the current CUDA device."""

    def __init__(self, model, weights: np.ndarray, stream=None, precision: int = PREC_FP32):
        import torch
        self._L = load()
        self.model = model
        cfg = Config(model.F, model.K, model.T, model.n_types, model.r_cut, model.gamma, precision)
        w = np.ascontiguousarray(weights, dtype=np.float32)
        if stream is None:
            stream = torch.cuda.current_stream()
        self._stream = stream
        h = C.c_void_p()
        st = self._L.sn_create(C.byref(cfg), w.ctypes.data, w.size, C.c_void_p(stream.cuda_stream), C.byref(h))
        if st != 0:
            raise SNError(st, "sn_create failed")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            self._L.sn_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != 0:
            raise SNError(st, self._L.sn_last_error(self._h).decode())

    def set_stream(self, stream):
        self._stream = stream
        self._check(self._L.sn_set_stream(self._h, C.c_void_p(stream.cuda_stream)))

    def reserve(self, system, max_edges: int):
        self._check(self._L.sn_reserve(self._h, C.byref(system_struct(system)), int(max_edges)))

    def build_neighbors(self, system, pos, row_ptr, col) -> int:
        """Fill row_ptr [N+1] / col [cap] (int32 CUDA tensors); returns E.  Raises SNError
        with status CAPACITY (and .needed = E) if col is too small."""
        import torch
        N = system.n_per_replica * system.n_replicas
        _dev_check(pos, torch.float32, "pos", 3 * N)
        _dev_check(row_ptr, torch.int32, "row_ptr", N + 1)
        _dev_check(col, torch.int32, "col")
        ne = C.c_int64(0)
        st = self._L.sn_build_neighbors(self._h, C.byref(system_struct(system)), _ptr(pos), _ptr(row_ptr),
                                        _ptr(col), col.numel(), C.byref(ne))
        if st == Status.CAPACITY:
            err = SNError(st, self._L.sn_last_error(self._h).decode())
            err.needed = ne.value
            raise err
        self._check(st)
        return ne.value

    def neighbors(self, system, pos, cap: int | None = None):
        """Convenience: allocate and return (row_ptr, col) for pos."""
        import torch
        N = system.n_per_replica * system.n_replicas
        row_ptr = torch.empty(N + 1, dtype=torch.int32, device=pos.device)
        cap = cap if cap is not None else max(64 * N, 1024)
        col = torch.empty(cap, dtype=torch.int32, device=pos.device)
        try:
            E = self.build_neighbors(system, pos, row_ptr, col)
        except SNError as e:
            if e.status != Status.CAPACITY:
                raise
            col = torch.empty(e.needed + 1, dtype=torch.int32, device=pos.device)
            E = self.build_neighbors(system, pos, row_ptr, col)
        return row_ptr, col[:E]

    def energy_forces(self, system, pos, types, row_ptr, col, energy=None, forces=None):
        import torch
        N = system.n_per_replica * system.n_replicas
        if energy is None:
            energy = torch.empty(system.n_replicas, dtype=torch.float32, device=pos.device)
        if forces is None:
            forces = torch.empty((N, 3), dtype=torch.float32, device=pos.device)
        R = system.n_replicas
        for t, dt, n, k in ((pos, torch.float32, "pos", 3 * N), (types, torch.int32, "types", N),
                            (row_ptr, torch.int32, "row_ptr", N + 1), (energy, torch.float32, "energy", R),
                            (forces, torch.float32, "forces", 3 * N)):
            _dev_check(t, dt, n, k)
        if col.numel():
            _dev_check(col, torch.int32, "col")
        self._check(self._L.sn_energy_forces(self._h, C.byref(system_struct(system)), _ptr(pos), _ptr(types),
                                             _ptr(row_ptr), _ptr(col), int(col.numel()), _ptr(energy),
                                             _ptr(forces)))
        return energy, forces

    def md_step(self, system, pos, vel, forces, types, mass: float, dt: float, n_steps: int,
                energy, kinetic):
        import torch
        _check_md_arrays(system, pos, vel, forces, types, energy, kinetic)
        self._check(self._L.sn_md_step(self._h, C.byref(system_struct(system)), _ptr(pos), _ptr(vel),
                                       _ptr(forces), _ptr(types), float(mass), float(dt), int(n_steps),
                                       _ptr(energy), _ptr(kinetic)))

    def md_langevin(self, system, pos, vel, forces, types, mass: float, dt: float, n_steps: int,
                    temperature: float, friction: float, seed: int, step0: int, energy, kinetic):
        """BAOAB Langevin steps (see sn_md_langevin); friction in 1/fs."""
        import torch
        _check_md_arrays(system, pos, vel, forces, types, energy, kinetic)
        self._check(self._L.sn_md_langevin(self._h, C.byref(system_struct(system)), _ptr(pos), _ptr(vel),
                                           _ptr(forces), _ptr(types), float(mass), float(dt), int(n_steps),
                                           float(temperature), float(friction), C.c_uint64(seed),
                                           C.c_int64(step0), _ptr(energy), _ptr(kinetic)))

    def md_step_host(self, system, pos, vel, forces, types, mass: float, dt: float, n_steps: int,
                     energy, kinetic):
        """Host-memory variant: numpy arrays or CPU (ideally pinned) torch tensors, updated
        in place."""
        self._check(self._L.sn_md_step_host(self._h, C.byref(system_struct(system)), _ptr(pos), _ptr(vel),
                                            _ptr(forces), _ptr(types), float(mass), float(dt), int(n_steps),
                                            _ptr(energy), _ptr(kinetic)))

    def sync(self):
        self._check(self._L.sn_sync(self._h))

    def set_wait_limit(self, cycles: int):
        """Bound (GPU clock cycles) of the tensor-core kernels' waits for their own MMAs; 0
        restores the default.  A tiny bound exercises the time-out path (see sn.h)."""
        self._check(self._L.sn_set_wait_limit(self._h, int(cycles)))

    def trace(self, on: bool = True):
        """Enable/disable per-kernel CUDA-event timing (see sn_trace_enable)."""
        self._check(self._L.sn_trace_enable(self._h, 1 if on else 0))

    def trace_read(self) -> dict:
        """{kernel class: (launches, total ms)} since the last read; synchronises."""
        buf = (TraceEntry * 32)()
        n = self._L.sn_trace_read(self._h, buf, 32)
        if n < 0:
            raise SNError(Status.CUDA, "sn_trace_read failed")
        return {buf[q].name.decode(): (int(buf[q].launches), float(buf[q].total_ms)) for q in range(min(n, 32))}

    def md_edges(self) -> int:
        return int(self._L.sn_md_edges(self._h))


def build_neighbors_noalloc(system, r_cut: float, pos, row_ptr, col, stream=None) -> int:
    """Neighbour list through sn_build_neighbors_noalloc, for callers that cannot allocate
    device memory: the library uses only its static scratch, the caller provides pos, row_ptr
    [N+1] and col [cap] (int32 CUDA tensors).  Returns E; raises SNError (with .needed on
    CAPACITY)."""
    import torch
    L = load()
    N = system.n_per_replica * system.n_replicas
    _dev_check(pos, torch.float32, "pos", 3 * N)
    _dev_check(row_ptr, torch.int32, "row_ptr", N + 1)
    _dev_check(col, torch.int32, "col")
    if stream is None:
        stream = torch.cuda.current_stream()
    ne = C.c_int64(0)
    st = L.sn_build_neighbors_noalloc(C.byref(system_struct(system)), float(r_cut), _ptr(pos), _ptr(row_ptr),
                                      _ptr(col), col.numel(), C.byref(ne), C.c_void_p(stream.cuda_stream))
    if st != 0:
        err = SNError(st, "sn_build_neighbors_noalloc failed")
        err.needed = ne.value
        raise err
    return ne.value


def version() -> str:
    return load().sn_version().decode()
