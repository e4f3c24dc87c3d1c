"""Replayed solves (mpq_params.solve_graphs): the second identical call of
mpq_solve captures its kernel launches into a CUDA graph and later calls
replay it.  The results must equal direct launches bit for bit (same kernels
in the same order), follow new contents of the same buffers, and count the
same kernel launches."""
import pytest
import torch

import mpq_inputs as mi
from tests.helpers import cu, spectrum_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mpq():
    import post_weight_quantization_row_b200 as m
    return m


def outputs(m, B, n):
    return {"idx": torch.empty(m, B, dtype=torch.int16, device="cuda"),
            "w_hat": torch.empty(m, n, dtype=torch.float32, device="cuda"),
            "energy": torch.empty(m, dtype=torch.float32, device="cuda")}


@pytest.mark.parametrize("kind", ["scalar", "vector"])
def test_graph_replay_equals_direct_launches(mpq, kind):
    if kind == "scalar":
        p = mi.small_problem(701, 40, 384, 600, d=1, levels=8, T_vamp=4, cd_sweeps=3)
    else:  # lattice codebook: tensor-core denoiser and CD scan, stream-ordered scratch
        cb = mi.e8_codebook_cached()[:512]
        p = mi.small_problem(702, 12, 160, 320, d=8, levels=512, T_vamp=3, cd_sweeps=2,
                             codebook=cb)
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    kw = {"codebook": p.codebook if p.d == 8 else None}
    pg = mpq.Plan.from_spectrum(s_cu, V_cu, p.d, p.levels, **kw)
    pd = mpq.Plan.from_spectrum(s_cu, V_cu, p.d, p.levels, solve_graphs=0, **kw)
    B = p.n // p.d
    W = cu(p.W)
    og, od = outputs(p.m_out, B, p.n), outputs(p.m_out, B, p.n)
    pd.solve(W, p.T_vamp, p.cd_sweeps, out=od)
    torch.cuda.synchronize()
    counts = []
    for _ in range(3):  # direct, capture + replay, replay
        for v in og.values():
            v.zero_()
        c0 = mpq.kernel_launch_count()
        pg.solve(W, p.T_vamp, p.cd_sweeps, out=og)
        torch.cuda.synchronize()
        counts.append(mpq.kernel_launch_count() - c0)
        for k in og:
            assert torch.equal(og[k], od[k]), k
    assert counts[0] == counts[1] == counts[2] > 0
    # new contents of the same buffer: the replay reads them
    W.copy_(W.flip(0))
    pd.solve(W, p.T_vamp, p.cd_sweeps, out=od)
    pg.solve(W, p.T_vamp, p.cd_sweeps, out=og)
    torch.cuda.synchronize()
    for k in og:
        assert torch.equal(og[k], od[k]), k
