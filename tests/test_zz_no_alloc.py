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
