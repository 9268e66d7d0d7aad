"""Pins of the oracle's neighbour list (CPU only).

The list is defined as every directed pair (j -> i), i != j, of the same replica whose fp32
squared distance (minimum image on periodic axes) is below r_cut^2; CSR rows by destination,
sources ascending inside a row.  These tests check the oracle's brute force against an
independent numpy float32 all-pairs evaluation, its cell list against its brute force, and
the properties the definition fixes (symmetry, exclusions, the strict cutoff).
"""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth


def numpy_pairs(pos, n_per, n_rep, box, r_cut):
    """All-pairs reference in numpy float32, one IEEE operation at a time (numpy does not
    contract to FMA)."""
    pos = pos.astype(np.float32)
    box = np.asarray(box, dtype=np.float32)
    rc2 = np.float32(r_cut) * np.float32(r_cut)
    rows = []
    for r in range(n_rep):
        P = pos[r * n_per:(r + 1) * n_per]
        d = P[None, :, :] - P[:, None, :]          # d[i, j] = x_j - x_i
        for a in range(3):
            if box[a] > 0:
                q = np.rint(d[..., a] / box[a]).astype(np.float32)
                d[..., a] = d[..., a] - box[a] * q
        xx = d[..., 0] * d[..., 0]
        yy = d[..., 1] * d[..., 1]
        zz = d[..., 2] * d[..., 2]
        r2 = (xx + yy) + zz
        m = r2 < rc2
        np.fill_diagonal(m, False)
        for i in range(n_per):
            rows.append(np.nonzero(m[i])[0].astype(np.int32) + r * n_per)
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(x) for x in rows])
    col = np.concatenate(rows) if rows else np.zeros(0, np.int32)
    return row_ptr, col


CASES = [
    ("chain32", synth.SystemCfg(32, 1), 10.0, "rw", 11),
    ("chains3x57", synth.SystemCfg(57, 3), 12.0, "saw", 12),
    ("box200", synth.SystemCfg(200, 1, (14.0, 14.0, 14.0)), 4.5, "box", 13),
    ("box2rep", synth.SystemCfg(150, 2, (16.0, 16.0, 16.0)), 5.0, "box", 14),
    ("box_aniso", synth.SystemCfg(300, 1, (15.5, 21.0, 31.0)), 5.0, "box", 15),
    ("tiny_box_fallback", synth.SystemCfg(40, 1, (9.0, 9.0, 9.0)), 4.0, "box", 16),
]


@pytest.mark.parametrize("name,system,r_cut,kind,seed", CASES, ids=[c[0] for c in CASES])
def test_brute_matches_numpy_all_pairs(oracle, name, system, r_cut, kind, seed):
    model = synth.ModelCfg(F=8, K=4, T=1, n_types=3, r_cut=r_cut)
    w = synth.make_custom(model, system, seed, kind)
    rp, cl = oracle.neighbors(system, r_cut, w.pos, "brute")
    rp2, cl2 = numpy_pairs(w.pos, system.n_per_replica, system.n_replicas, system.box, r_cut)
    assert np.array_equal(rp, rp2)
    assert np.array_equal(cl, cl2)
    assert len(cl) > 0


@pytest.mark.parametrize("name,system,r_cut,kind,seed",
                         [c for c in CASES if c[1].periodic], ids=[c[0] for c in CASES if c[1].periodic])
def test_cells_equal_brute(oracle, name, system, r_cut, kind, seed):
    model = synth.ModelCfg(F=8, K=4, T=1, n_types=3, r_cut=r_cut)
    w = synth.make_custom(model, system, seed, kind)
    rp, cl = oracle.neighbors(system, r_cut, w.pos, "brute")
    rp2, cl2 = oracle.neighbors(system, r_cut, w.pos, "cells")
    assert np.array_equal(rp, rp2) and np.array_equal(cl, cl2)


def test_cells_equal_brute_config4_and_unwrapped(oracle):
    w = synth.make_workload(4)
    s = w.system
    rp, cl = oracle.neighbors(s, w.model.r_cut, w.pos, "brute")
    rp2, cl2 = oracle.neighbors(s, w.model.r_cut, w.pos, "cells")
    assert np.array_equal(rp, rp2) and np.array_equal(cl, cl2)
    # the list is the same set for coordinates shifted by whole box lengths only up to
    # fp32 rounding of the shifted coordinates; the cell list must still equal brute force
    shifted = (w.pos + np.float32(40.6) * np.array([1, -2, 3], np.float32)).astype(np.float32)
    rp3, cl3 = oracle.neighbors(s, w.model.r_cut, shifted, "brute")
    rp4, cl4 = oracle.neighbors(s, w.model.r_cut, shifted, "cells")
    assert np.array_equal(rp3, rp4) and np.array_equal(cl3, cl4)


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_list_properties(oracle, cfg):
    w = synth.make_workload(cfg)
    s = w.system
    rp, cl = oracle.neighbors(s, w.model.r_cut, w.pos, "cells" if s.periodic else "brute")
    N = s.n_atoms
    dst = np.repeat(np.arange(N), np.diff(rp))
    # no self edges, no cross-replica edges, rows sorted strictly ascending
    assert np.all(dst != cl)
    assert np.all(dst // s.n_per_replica == cl // s.n_per_replica)
    for i in range(0, N, max(1, N // 500)):
        row = cl[rp[i]:rp[i + 1]]
        assert np.all(np.diff(row) > 0)
    # symmetric: j -> i exists iff i -> j exists
    a = set(zip(dst.tolist(), cl.tolist()))
    b = set(zip(cl.tolist(), dst.tolist()))
    assert a == b


def test_strict_cutoff_and_exclusions(oracle):
    box0 = (0.0, 0.0, 0.0)
    # r^2 == r_c^2 exactly in fp32 (4 = 2*2): not an edge; just inside: an edge
    assert not oracle.pair_within([0, 0, 0], [2, 0, 0], box0, 2.0)
    assert oracle.pair_within([0, 0, 0], [np.nextafter(np.float32(2), np.float32(0)), 0, 0], box0, 2.0)
    # periodic minimum image: 0.5 and 9.7 in a 10 A box are 0.8 apart
    assert oracle.pair_within([0.5, 0, 0], [9.7, 0, 0], (10.0, 10.0, 10.0), 1.0)
    assert not oracle.pair_within([0.5, 0, 0], [9.7, 0, 0], box0, 1.0)
    # coincident atoms of different index are an edge (d = 0 < r_c)
    s = synth.SystemCfg(3, 1)
    pos = np.array([[0, 0, 0], [0, 0, 0], [50, 0, 0]], np.float32)
    rp, cl = oracle.neighbors(s, 5.0, pos)
    assert rp.tolist() == [0, 1, 2, 2] and cl.tolist() == [1, 0]


def test_empty_and_isolated(oracle):
    s = synth.SystemCfg(0, 1)
    rp, cl = oracle.neighbors(s, 5.0, np.zeros((0, 3), np.float32))
    assert rp.tolist() == [0] and cl.size == 0
    s = synth.SystemCfg(1, 4)
    rp, cl = oracle.neighbors(s, 5.0, np.zeros((4, 3), np.float32))   # one atom per replica
    assert rp.tolist() == [0, 0, 0, 0, 0] and cl.size == 0


def test_rejects_cutoff_beyond_half_box(oracle):
    s = synth.SystemCfg(10, 1, (9.0, 9.0, 9.0))
    with pytest.raises(ValueError):
        oracle.neighbors(s, 4.5, np.zeros((10, 3), np.float32))
