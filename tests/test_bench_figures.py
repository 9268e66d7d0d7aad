"""The derived figures of the benchmark line, checked on the CPU: the whole-evaluation roofline
(the path's filter FLOPs and compulsory HBM bytes, the slower of the two roofs), the NVE drift
statistics of cfg3, and the look-up of the profiled DRAM traffic of the dominant kernel."""
import hashlib
import importlib.util
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_figures_module", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class Model:
    F, K, T = 128, 50, 3


PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1646.8, "bf16_tflops_sustained": 1398.0}


def test_eval_roofline_counts(bench):
    N, E, t = 17216, 292756.0, 656e-6
    r = bench.eval_roofline(Model, N, E, t, PEAKS)
    # per directed edge and block: forward K->F and F->F, backward F->F and F->K, two flops
    # per multiply-add; cfg2's 292,756 edges over 3 blocks give 8.0e10
    assert r["flops"] == pytest.approx(2 * 2 * (50 * 128 + 128 * 128) * E * 3)
    assert r["flops"] == pytest.approx(8.004e10, rel=1e-3)
    # per block eight passes over an [N][F] fp32 array and two 4-byte indices per edge;
    # positions (12 B), types (4 B) and forces (12 B) once per evaluation
    nbytes = 8 * N * 128 * 4 * 3 + 8 * E * 3 + (12 + 4 + 12) * N
    assert r["bytes"] == pytest.approx(nbytes)
    t_tc, t_hbm = r["flops"] / 1398e12, nbytes / 6551e9
    assert r["bound"] == "tensor" and t_tc > t_hbm
    assert r["t_roof_us"] == pytest.approx(t_tc * 1e6)
    assert r["frac"] == pytest.approx(t_tc / t)
    assert r["edges_per_s"] == pytest.approx(E / t)
    # an MD step adds the list build and the integrator: 80 bytes per atom, the 4-byte col per edge
    rb = bench.eval_roofline(Model, N, E, t, PEAKS, build=True)
    assert rb["bytes"] - r["bytes"] == pytest.approx(80 * N + 4 * E)
    # without edges the roof is the HBM one
    r0 = bench.eval_roofline(Model, N, 0.0, t, PEAKS)
    assert r0["bound"] == "hbm" and r0["flops"] == 0.0
    assert r0["t_roof_us"] == pytest.approx((8 * N * 128 * 4 * 3 + 28 * N) / 6551e9 * 1e6)


def test_drift_figures_of_a_linear_drift(bench):
    # two replicas whose total energy grows linearly by a and 3a per step
    n_per, steps, a = 269, 10, 0.01
    k = np.arange(steps + 1, dtype=np.float64)[:, None]
    etot = 100.0 + np.array([[a, 3 * a]]) * k
    fig = bench.drift_figures(etot, n_per, steps)
    nkT = n_per * bench.synth.KB * bench.TEMP
    assert fig["steps"] == steps and fig["dt_fs"] == bench.DT
    assert fig["max_abs_drift_per_nkT"]["max"] == pytest.approx(3 * a * steps / nkT)
    assert fig["max_abs_drift_per_nkT"]["median"] == pytest.approx(2 * a * steps / nkT)
    # the replica mean grows by 2a per step of DT fs: per ns that is 2a / nkT / (DT * 1e-6)
    assert fig["slope_per_ns_per_nkT"] == pytest.approx(2 * a / nkT / (bench.DT * 1e-6))


def test_traffic_lookup_follows_the_kernel_source(bench, tmp_path):
    src = ROOT / "schnet_gnn_molecular_cell_b200" / "csrc" / "sn_ef_tc.cu"
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    recorded = [l.split() for l in (ROOT / "profiles" / "traffic.txt").read_text().splitlines()
                if l.startswith("edge_bwd ")]
    assert recorded, "no edge_bwd entry"
    fields = dict(kv.split("=", 1) for kv in recorded[0][1:])
    value = bench.kernel_traffic("edge_bwd", src, fields["precision"])
    if fields["src"] == sha:   # taken on the current source: reported
        assert value == float(fields["bytes_per_launch"])
    else:                      # the kernel changed since: not reported
        assert value is None
    # another precision or kernel has no entry
    assert bench.kernel_traffic("edge_bwd", src, "tc32") is None
    assert bench.kernel_traffic("edge_fwd", src, "fp16") is None
    # a different source text never matches
    other = tmp_path / "sn_ef_tc.cu"
    other.write_bytes(src.read_bytes() + b"\n")
    assert bench.kernel_traffic("edge_bwd", other, fields["precision"]) is None
