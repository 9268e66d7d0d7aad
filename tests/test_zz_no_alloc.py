"""The neighbour-list entry point that allocates nothing, for callers that cannot call
cudaMalloc (an engine that has reserved the device memory for its own pool, a step loop
that must not pay cudaMalloc's implicit synchronisation, a host application that forbids
allocations it does not own).

It must give exactly the list of the allocating entry point (sn_build_neighbors through a
context), call after call: its scratch is one static device array shared by every call, so
a second call must not see leftovers of the first.  The test allocates the inputs and
outputs itself (torch); the entry point under test only uses its static array.

This file is collected last on purpose, so that a run stopping at the first failure has run
every other test before it.
"""
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


def _allocating_list(w, dev):
    from schnet_gnn_molecular_cell_b200 import Context
    ctx = Context(w.model, w.weights)
    rp, cl = ctx.neighbors(w.system, torch.from_numpy(w.pos).to(dev))
    ctx.sync()
    return rp.cpu().numpy(), cl.cpu().numpy()


def _noalloc_list(w, dev, cap):
    from schnet_gnn_molecular_cell_b200.binding import build_neighbors_noalloc
    N = w.system.n_atoms
    pos = torch.from_numpy(w.pos).to(dev)
    row_ptr = torch.full((N + 1,), -7, dtype=torch.int32, device=dev)
    col = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    E = build_neighbors_noalloc(w.system, w.model.r_cut, pos, row_ptr, col)
    torch.cuda.synchronize()
    return row_ptr.cpu().numpy(), col[:E].cpu().numpy()


def test_noalloc_equals_allocating_builder_on_consecutive_calls(dev):
    # periodic box (cell list), then open chains (all pairs), then the box again: each call
    # must match the allocating builder exactly (integer output: bit for bit)
    box = synth.make_workload(4)
    chains = synth.make_workload(2)
    for w in (box, chains, box):
        rp_a, cl_a = _allocating_list(w, dev)
        rp_n, cl_n = _noalloc_list(w, dev, cap=len(cl_a) + 1000)
        assert np.array_equal(rp_n, rp_a)
        assert np.array_equal(cl_n, cl_a)


def test_noalloc_reports_capacity_and_rejects_oversize(dev):
    from schnet_gnn_molecular_cell_b200 import SNError, Status
    from schnet_gnn_molecular_cell_b200.binding import build_neighbors_noalloc
    w = synth.make_workload(1)
    rp_a, cl_a = _allocating_list(w, dev)
    pos = torch.from_numpy(w.pos).to(dev)
    row_ptr = torch.empty(33, dtype=torch.int32, device=dev)
    small = torch.empty(8, dtype=torch.int32, device=dev)
    with pytest.raises(SNError) as ei:
        build_neighbors_noalloc(w.system, w.model.r_cut, pos, row_ptr, small)
    assert ei.value.status == Status.CAPACITY and ei.value.needed == len(cl_a)
    big = synth.SystemCfg(65537, 1)
    with pytest.raises(SNError) as ei:
        build_neighbors_noalloc(big, 5.0, torch.zeros((65537, 3), device=dev),
                                torch.empty(65538, dtype=torch.int32, device=dev),
                                torch.empty(16, dtype=torch.int32, device=dev))
    assert ei.value.status == Status.UNSUPPORTED
    # still correct after the rejected calls
    rp_n, cl_n = _noalloc_list(w, dev, cap=len(cl_a))
    assert np.array_equal(rp_n, rp_a) and np.array_equal(cl_n, cl_a)


def test_noalloc_rejects_short_arrays_before_any_launch(dev):
    # a row_ptr one entry short, or too few positions, is refused by the binding with
    # INVALID_ARG before the library (and any kernel) sees the pointers
    from schnet_gnn_molecular_cell_b200 import SNError, Status
    from schnet_gnn_molecular_cell_b200.binding import build_neighbors_noalloc
    w = synth.make_workload(1)
    N = w.system.n_atoms
    pos = torch.from_numpy(w.pos).to(dev)
    col = torch.empty(4096, dtype=torch.int32, device=dev)
    with pytest.raises(SNError) as ei:
        build_neighbors_noalloc(w.system, w.model.r_cut, pos, torch.empty(N, dtype=torch.int32, device=dev), col)
    assert ei.value.status == Status.INVALID_ARG
    with pytest.raises(SNError) as ei:
        build_neighbors_noalloc(w.system, w.model.r_cut, pos[: N - 1], torch.empty(N + 1, dtype=torch.int32,
                                                                                  device=dev), col)
    assert ei.value.status == Status.INVALID_ARG
