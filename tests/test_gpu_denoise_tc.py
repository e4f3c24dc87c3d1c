"""Parity of the vector (d = 8) denoiser on both engines with the float64
oracle: the tensor-core kernel (lattice codebooks: scores on tcgen05, moments
centred on the argmax) and the SIMT kernel (any codebook).

Cases span several 128-block tiles with a ragged tail, the persistent loop
(more 128-block tiles than SMs), the anchored prior, the hard limit (huge
precision: the posterior is a point mass on the nearest codeword), the
nearest-codeword init, and codebooks that do not qualify for the tensor
cores.  Bars as in the other stage tests: per-row relative l2 1e-4 for
x_hat and the block variances, 1e-4 on the per-row sums; indices exact
except where the oracle's top-two logit gap is below 1e-3."""
import math

import numpy as np
import pytest
import torch

import mpq_inputs as mi
from oracle import mpq_oracle as orc
from tests.helpers import (assert_vec_close, assert_rows_close, assert_scalars_close, codebook_for, cu, host,
                           idx_np, injected_state, spectrum_cuda)

pytestmark = pytest.mark.gpu

LOGIT_TIE = 1e-3
ENGINES = {"simt": 1, "tensor": 2}


@pytest.fixture(scope="module")
def mpq():
    import post_weight_quantization_row_b200 as m
    return m


def e8_case(seed, m_out, n, K, m=None):
    cb = mi.e8_codebook_cached()[:K]
    return mi.small_problem(seed, m_out, n, m or 2 * n, d=8, levels=K, T_vamp=4, cd_sweeps=3,
                            codebook=cb)


def plan_for(mpq, p, engine, tau=math.inf, **kw):
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    return mpq.Plan.from_spectrum(s_cu, V_cu, 8, p.levels, codebook=p.codebook,
                                  vec_engine=ENGINES[engine], tau=tau, **kw)


def kernels_of(mpq, fn):
    mpq.profile_start()
    out = fn()
    torch.cuda.synchronize()
    return out, mpq.profile_stop()


def check_denoise(mpq, p, plan, R1, g1, engine, tau=math.inf):
    """Stage parity of the vector denoiser; the plan's anchor must be tau."""
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    off = np.zeros_like(sc)
    anchored = math.isfinite(tau)
    ref = orc.denoise(R1, g1, codebook_for(p), sc.astype(np.float64), off.astype(np.float64),
                      p.W, tau)
    out, kern = kernels_of(mpq, lambda: plan.stage_denoise(
        cu(R1), cu(g1, torch.float64), cu(sc), cu(off), cu(p.W) if anchored else None))
    want = "k_denoise_vec_tc" if engine == "tensor" else "k_denoise_vec"
    assert want in kern, kern
    assert_vec_close("xhat1", host(out["xhat"]), ref.xhat)
    assert_vec_close("vblock", host(out["vblock"]), ref.vblock)
    assert_scalars_close("vsum", host(out["vsum"]), ref.vsum)
    ok = ref.gap > LOGIT_TIE
    assert ok.mean() > 0.9
    assert np.array_equal(idx_np(out["idx"])[ok], ref.idx[ok])
    return out, ref


@pytest.mark.parametrize("engine", ["tensor", "simt"])
@pytest.mark.parametrize("g_lo,g_hi", [(0.3, 3.0), (1.0, 30.0), (30.0, 3000.0)])
def test_denoise_e8_ragged_tiles(mpq, engine, g_lo, g_hi):
    # 21 rows x 20 blocks = 420 blocks: three full 128-block tiles + 36
    p = e8_case(202, 21, 160, 2048)
    plan = plan_for(mpq, p, engine)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    s, _ = orc.spectrum(p.X)
    R1, g1, _, _, _, _ = injected_state(8, p.W, sc, s, g_lo, g_hi)
    check_denoise(mpq, p, plan, R1, g1, engine)


@pytest.mark.parametrize("engine", ["tensor", "simt"])
@pytest.mark.parametrize("tau", [0.2, 0.7])
def test_denoise_e8_anchored_prior(mpq, engine, tau):
    p = e8_case(203, 13, 96, 1024)
    plan = plan_for(mpq, p, engine, tau=tau)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    s, _ = orc.spectrum(p.X)
    R1, g1, _, _, _, _ = injected_state(9, p.W, sc, s)
    check_denoise(mpq, p, plan, R1, g1, engine, tau=tau)


def test_denoise_e8_persistent_tiles(mpq):
    # 300 rows x 64 blocks = 19200 blocks = 150 tiles of 128: more tiles than
    # SMs, so CTAs walk several tiles and the pipelines carry over
    p = e8_case(204, 300, 512, 256, m=600)
    plan = plan_for(mpq, p, "tensor")
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    s, _ = orc.spectrum(p.X)
    R1, g1, _, _, _, _ = injected_state(10, p.W, sc, s)
    check_denoise(mpq, p, plan, R1, g1, "tensor")


@pytest.mark.parametrize("engine", ["tensor", "simt"])
def test_denoise_hard_limit_is_nearest_codeword(mpq, engine):
    # gamma1 s^2 = 1e12: the posterior is a point mass on the nearest codeword
    p = e8_case(205, 9, 64, 512)
    plan = plan_for(mpq, p, engine)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    R1 = p.W.astype(np.float32)
    g1 = 1e12 / (sc.astype(np.float64) ** 2)
    cb = codebook_for(p)
    out = plan.stage_denoise(cu(R1), cu(g1, torch.float64), cu(sc), cu(np.zeros_like(sc)))
    t = R1.astype(np.float64) / sc[:, None].astype(np.float64)
    nn = orc.nearest_codewords(t, cb).reshape(p.m_out, -1)
    d2 = ((t.reshape(-1, 8)[:, None, :] - cb[None]) ** 2).sum(-1)
    two = np.partition(d2, 1, axis=1)[:, :2]
    ok = ((two[:, 1] - two[:, 0]) > 1e-5 * two[:, 1]).reshape(p.m_out, -1)
    assert ok.mean() > 0.95
    got = idx_np(out["idx"])
    assert np.array_equal(got[ok], nn[ok])
    # x_hat decodes the device's own argmax exactly; no posterior spread
    dec = orc.decode(got, cb, sc.astype(np.float64), np.zeros(p.m_out))
    assert np.allclose(host(out["xhat"]), dec, rtol=1e-6, atol=1e-7)
    assert np.all(host(out["vblock"]) == 0.0)


@pytest.mark.parametrize("engine", ["tensor", "simt"])
def test_init_nearest_codeword(mpq, engine):
    p = e8_case(206, 17, 200, 1024)
    plan = plan_for(mpq, p, engine)
    out, kern = kernels_of(mpq, lambda: plan.stage_init(cu(p.W)))
    assert ("k_denoise_vec_tc(nearest)" in kern) == (engine == "tensor"), kern
    sc = host(out["scale"]).astype(np.float64)
    cb = codebook_for(p)
    st = orc.init(p.W, cb, sc, np.zeros_like(sc))
    got = idx_np(out["idx"])
    for i in range(p.m_out):
        blocks = p.W[i].reshape(-1, 8).astype(np.float64) / sc[i]
        d2 = ((blocks[:, None, :] - cb[None]) ** 2).sum(-1)
        two = np.partition(d2, 1, axis=1)[:, :2]
        ok = (two[:, 1] - two[:, 0]) > 1e-5 * two[:, 1]
        assert np.array_equal(got[i][ok], st.idx_rtn[i][ok])


def test_auto_engine_picks_tensor_cores_for_lattice_codebooks(mpq):
    p = e8_case(207, 5, 64, 256)
    plan = plan_for(mpq, p, "tensor")
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    auto = mpq.Plan.from_spectrum(s_cu, V_cu, 8, p.levels, codebook=p.codebook, tau=math.inf)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    args = (cu(p.W), cu(np.full(p.m_out, 5.0) / sc.astype(np.float64) ** 2, torch.float64),
            cu(sc), cu(np.zeros_like(sc)))
    a, kern = kernels_of(mpq, lambda: auto.stage_denoise(*args))
    assert "k_denoise_vec_tc" in kern
    b = plan.stage_denoise(*args)
    assert torch.equal(a["xhat"], b["xhat"]) and torch.equal(a["idx"], b["idx"])


@pytest.mark.parametrize("codebook", ["gaussian", "ragged_K"])
def test_codebooks_that_do_not_qualify(mpq, codebook):
    g = np.random.default_rng(11)
    if codebook == "gaussian":   # coordinates not on a dyadic grid
        cb = g.standard_normal((256, 8)).astype(np.float32)
    else:                        # K not a multiple of 128
        cb = mi.e8_codebook_cached()[:200]
    p = mi.small_problem(208, 7, 64, 128, d=8, levels=cb.shape[0], codebook=cb)
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    with pytest.raises(mpq.MPQError) as e:
        mpq.Plan.from_spectrum(s_cu, V_cu, 8, p.levels, codebook=cb, vec_engine=2)
    assert e.value.status == 7   # MPQ_ERR_UNSUPPORTED
    # the default engine falls back to the SIMT kernel and matches the oracle
    plan = mpq.Plan.from_spectrum(s_cu, V_cu, 8, p.levels, codebook=cb, tau=math.inf)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    s, _ = orc.spectrum(p.X)
    R1, g1, _, _, _, _ = injected_state(12, p.W, sc, s)
    check_denoise(mpq, p, plan, R1, g1, "simt")


@pytest.mark.parametrize("engine", ["tensor", "simt"])
@pytest.mark.parametrize("tau", [math.inf, orc.TAU])
def test_vector_solve_both_engines(mpq, engine, tau):
    p = e8_case(209, 23, 160, 2048, m=320)
    plan = plan_for(mpq, p, engine, tau=tau)
    out = plan.solve(cu(p.W), p.T_vamp, p.cd_sweeps, stats=True)
    s, V = orc.spectrum(p.X)
    ref = orc.solve(p.W, codebook_for(p), s, V, p.T_vamp, p.cd_sweeps, tau=tau)
    e_gpu = host(out["energy"]).astype(np.float64)
    rel = np.abs(e_gpu - ref.energy) / ref.energy
    clean = np.all(ref.map_gap > 1e-4, axis=1) & (ref.cd.first_tie < 0)
    assert clean.mean() >= 0.25
    assert np.array_equal(idx_np(out["idx"])[clean], ref.idx[clean])
    assert rel[clean].max() <= 1e-3
    assert rel.max() <= 5e-2 and np.mean((e_gpu - ref.energy) / ref.energy) <= 1e-2


@pytest.mark.parametrize("g_lo,g_hi,tau", [(0.3, 3.0, math.inf), (3.0, 30.0, math.inf),
                                           (30.0, 300.0, math.inf), (300.0, 3000.0, math.inf),
                                           (3.0, 30.0, orc.TAU)])
def test_denoise_full_e8_codebook_on_e8t8_rows(mpq, g_lo, g_hi, tau):
    # the whole 65536-codeword offset-E8 codebook (every shell up to norm^2
    # 11.5, all 512 codebook stages of the kernel's ring) on two rows of the
    # 2-bit workload (1024 blocks, 8 tiles of 128), precisions gamma1 s^2
    # from 0.3 to 3000; the denoiser reads no spectrum, so the plan takes a
    # small synthetic one
    p = mi.make_problem("e8t8", rows=[11, 12], with_x=False)
    s, V = mi.orthonormal_spectrum(31, p.n, 64)
    plan = mpq.Plan.from_spectrum(cu(s, torch.float64), cu(V, torch.float64), 8, p.levels,
                                  codebook=p.codebook, tau=tau)
    sc = orc.rms_scale(p.W)[0].astype(np.float32)
    R1, g1, _, _, _, _ = injected_state(13, p.W, sc, s, g_lo, g_hi)
    check_denoise(mpq, p, plan, R1, g1, "tensor", tau=tau)
