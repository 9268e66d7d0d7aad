"""The device time-out path of the tensor-core kernels, made to run out on purpose.

Every wait of these kernels is for their own MMAs and is bounded; sn_set_wait_limit shortens
the bound of the MMA waits far below an MMA's duration, so that the first wait gives up.  The
kernel must report SN_ERR_TIMEOUT through sn_sync, let its issued MMAs finish before releasing
tensor memory, and leave the context usable: the next call with the default bound gives the
same result, bit for bit, as a context that never timed out, within the mode's tolerance of
the oracle.  Nothing here faults or hangs: the waits are bounded either way.
"""
import numpy as np
import pytest

from schnet_gnn_molecular_cell_b200 import synth
from tests.test_gpu_parity import assert_close, to_dev
from tests.test_gpu_tensor import assert_close16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.mark.parametrize("precision", [1, 2], ids=["fp16", "tc32"])
def test_mma_wait_times_out_and_the_context_recovers(oracle, dev, precision):
    from schnet_gnn_molecular_cell_b200 import Context, SNError, Status
    w = synth.make_workload(4)
    s, m = w.system, w.model
    pos, types = to_dev(w.pos, dev), to_dev(w.types, dev)
    ref = Context(m, w.weights, precision=precision)
    rp, cl = ref.neighbors(s, pos)
    E_ref, F_ref = ref.energy_forces(s, pos, types, rp, cl)
    ref.sync()

    ctx = Context(m, w.weights, precision=precision)
    ctx.set_wait_limit(1)                  # one cycle: the first MMA wait gives up
    ctx.energy_forces(s, pos, types, rp, cl)
    with pytest.raises(SNError) as ei:
        ctx.sync()
    assert ei.value.status == Status.TIMEOUT
    ctx.set_wait_limit(0)                  # default bound
    E, F = ctx.energy_forces(s, pos, types, rp, cl)
    ctx.sync()
    assert torch.equal(E, E_ref) and torch.equal(F, F_ref)
    rp_o, cl_o = oracle.neighbors(s, m.r_cut, w.pos, "cells")
    E_o, F_o, _ = oracle.energy_forces(m, w.weights, s, w.pos, w.types, rp_o, cl_o)
    check = assert_close16 if precision == 1 else assert_close
    check(E.cpu().numpy(), E_o, "energy after the time-out")
    check(F.cpu().numpy(), F_o, "forces after the time-out")


def test_md_step_times_out_in_the_pipelined_forward(dev):
    # the fp16 forward is the warp-specialised pipeline (bounded waits on its stage barriers):
    # an MD step with a one-cycle bound reports the time-out and the next step runs normally
    from schnet_gnn_molecular_cell_b200 import Context, SNError, Status
    w = synth.make_workload(2)
    s = w.system
    ctx = Context(w.model, w.weights, precision=1)
    pos = to_dev(w.pos.copy(), dev)
    vel = to_dev(synth.maxwell_boltzmann(s.n_per_replica, s.n_replicas, 12.0, 300.0, 4002), dev)
    types = to_dev(w.types, dev)
    rp, cl = ctx.neighbors(s, pos)
    _, forces = ctx.energy_forces(s, pos, types, rp, cl)
    forces = forces.clone()
    e = torch.empty(s.n_replicas, device=dev)
    k = torch.empty(s.n_replicas, device=dev)
    ctx.set_wait_limit(1)
    ctx.md_step(s, pos.clone(), vel.clone(), forces.clone(), types, 12.0, 2.0, 1, e, k)
    with pytest.raises(SNError) as ei:
        ctx.sync()
    assert ei.value.status == Status.TIMEOUT
    ctx.set_wait_limit(0)
    ctx.md_step(s, pos, vel, forces, types, 12.0, 2.0, 1, e, k)
    ctx.sync()
    assert torch.isfinite(e).all() and torch.isfinite(forces).all()


def test_negative_wait_limit_is_rejected(dev):
    from schnet_gnn_molecular_cell_b200 import Context, SNError, Status
    w = synth.make_workload(4)
    ctx = Context(w.model, w.weights, precision=1)
    with pytest.raises(SNError) as ei:
        ctx.set_wait_limit(-5)
    assert ei.value.status == Status.INVALID_ARG
