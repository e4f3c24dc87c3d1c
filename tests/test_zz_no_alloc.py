"""The allocation-free energy entry point (mpq_stage_energy_noalloc).

Callers whose device memory is owned by someone else -- a framework allocator
that holds the whole GPU, a serving loop that must not stall on the
synchronisation an allocation implies, a process with a fixed memory budget --
use this entry point instead of mpq_stage_energy.  Its scratch is one static
device array shared by every call, so these tests check that two calls in a
row (the second one on different, smaller inputs, with the first call's data
still in the array) give the same results as the workspace-backed entry
point, and that calls too large for the array are refused before anything is
launched.  This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

import mpq_inputs as mi
from oracle import mpq_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    import post_weight_quantization_row_b200 as mpq
    p = mi.small_problem(909, 48, 200, 300, d=1, levels=8)
    s, V = orc.spectrum(p.X)
    plan = mpq.Plan.from_spectrum(torch.from_numpy(s).cuda(), torch.from_numpy(V).cuda(), 1,
                                  p.levels)
    st = orc.init(p.W, orc.scalar_levels(p.levels))
    return mpq, p, plan, st


def _args(p, st, rows, seed):
    g = np.random.default_rng(seed)
    idx = g.integers(0, p.levels, size=(rows, p.n)).astype(np.uint16).view(np.int16)
    W = torch.from_numpy(p.W[:rows]).cuda()
    sc = torch.from_numpy(st.scale[:rows].astype(np.float32)).cuda()
    off = torch.from_numpy(st.offset[:rows].astype(np.float32)).cuda()
    return W, sc, off, torch.from_numpy(idx).cuda()


def test_noalloc_energy_matches_workspace_entry_point_twice(setup):
    mpq, p, plan, st = setup
    for rows, seed in ((48, 1), (17, 2)):  # second call: fewer rows, stale scratch beyond them
        W, sc, off, idx = _args(p, st, rows, seed)
        ref = plan.stage_energy(W, sc, off, idx)
        got = plan.stage_energy_noalloc(W, sc, off, idx)
        plan.status()
        assert torch.equal(got["w_hat"], ref["w_hat"])
        e_ref = ref["energy"].double()
        assert torch.all((got["energy"].double() - e_ref).abs() <= 1e-5 * e_ref)


def test_noalloc_refuses_calls_larger_than_its_array(setup):
    mpq, p, plan, st = setup
    per_row = 4 * plan.n + 4 * plan.r + 2 * plan.B
    rows = mpq._lib.NOALLOC_SCRATCH_BYTES // per_row + 1
    W = torch.zeros(rows, plan.n, dtype=torch.float32, device="cuda")
    sc = torch.ones(rows, dtype=torch.float32, device="cuda")
    idx = torch.zeros(rows, plan.B, dtype=torch.int16, device="cuda")
    before = mpq.kernel_launch_count()
    with pytest.raises(mpq.MPQError) as e:
        plan.stage_energy_noalloc(W, sc, torch.zeros_like(sc), idx)
    assert e.value.status == 1
    assert mpq.kernel_launch_count() == before


def test_noalloc_energy_allocates_nothing(setup):
    """On a fresh plan whose workspace cap (1 byte) makes any workspace
    allocation fail, the entry point still runs, and the device's free
    memory and torch's allocated bytes are the same before and after two
    calls (a first call runs before the measurement: loading the library's
    kernels on first use may reserve device memory once per process)."""
    mpq, p, _, st = setup
    s, V = orc.spectrum(p.X)
    plan = mpq.Plan.from_spectrum(torch.from_numpy(s).cuda(), torch.from_numpy(V).cuda(), 1,
                                  p.levels)
    plan.set_workspace_cap(1)
    W, sc, off, idx = _args(p, st, 40, 3)
    w_hat = torch.empty(40, plan.n, dtype=torch.float32, device="cuda")
    energy = torch.empty(40, dtype=torch.float32, device="cuda")
    plan.stage_energy_noalloc(W, sc, off, idx, w_hat, energy)
    plan.status()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch0 = torch.cuda.memory_allocated()
    for _ in range(2):
        plan.stage_energy_noalloc(W, sc, off, idx, w_hat, energy)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == torch0
    plan.status()
    # the workspace-backed entry point on the same plan needs workspace and
    # is refused by the cap, so the calls above never created any
    with pytest.raises(mpq.MPQError) as e:
        plan.stage_energy(W, sc, off, idx)
    assert e.value.status == 3
    e_ref = orc.energy(p.W[:40], orc.decode(idx.cpu().numpy().view(np.uint16).astype(np.int64),
                                             orc.scalar_levels(p.levels),
                                             sc.cpu().numpy().astype(np.float64),
                                             off.cpu().numpy().astype(np.float64)), s, V)
    got = energy.double().cpu().numpy()
    assert np.all(np.abs(got - e_ref) <= 1e-4 * e_ref)
    plan.close()
