"""GPU parity of the factor path (lf_tsqr_batched, lf_select_ranks,
lf_truncate_export) against the fp64 oracle on the same input bytes."""
import numpy as np
import pytest
import torch

from oracle import allocate as OA
from oracle import factor as OF
from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def upload(Bh, Ah):
    return Bh.cuda(), Ah.cuda()


def check_tsqr(layout, Bh, Ah, F, idx):
    rs = F.rs
    RB, RA, S = F.R_B.cpu().numpy(), F.R_A.cpu().numpy(), F.sigma.cpu().numpy()
    for i in idx:
        B, A = G.module_np(layout, Bh, Ah, i)
        r = B.shape[1]
        RBo, RAo = OF.qr_r(B), OF.qr_r(A.T)
        for got, want in ((RB[i][:r, :r], RBo), (RA[i][:r, :r], RAo)):
            assert np.allclose(np.tril(got, -1), 0)
            assert np.all(np.diag(got) >= 0)
            err = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
            assert err <= G.R_TOL, (i, err)
        assert np.all(RB[i][r:, :] == 0) and np.all(RB[i][:, r:] == 0)
        s, *_ = OF.spectrum_factor(B, A)
        assert np.max(np.abs(S[i][:r] - s)) <= G.SIGMA_TOL * max(s[0], 1e-300), i
        assert np.all(S[i][r:] == 0)
        assert np.all(np.diff(S[i][:r]) <= 0)


def test_tiny_tsqr_and_uniform_export():
    lay, Bh, Ah = synth.tiny_fleet()
    B, A = upload(Bh, Ah)
    mods, F, E, st = G.run_factor_path(lay, B, A, lf.policy_U(1, 4))
    assert st == 0
    check_tsqr(lay, Bh, Ah, F, range(lay.n))
    assert E.ranks.cpu().tolist() == [4, 4, 4, 4]
    offA = E.off_A.cpu().numpy()
    assert offA.tolist() == [0, 1024, 2048, 3072, 4096]
    sig = G.oracle_sigma_rows(lay, Bh, Ah, range(lay.n))
    for eg, eo in G.recon_errors(lay, Bh, Ah, E, sig, range(lay.n)):
        assert abs(eg - eo) <= G.RECON_TOL
    # definition route on the tiny case: dense SVD of B A
    for i in range(lay.n):
        Bn, An = G.module_np(lay, Bh, Ah, i)
        s_d, *_ = OF.spectrum_dense(Bn, An)
        assert np.allclose(F.sigma[i].cpu().numpy(), s_d, rtol=0, atol=G.SIGMA_TOL * s_d[0])
    # bf16 pools are the fp32 pools rounded once
    assert torch.equal(E.A_pool16[:4096], E.A_pool[:4096].to(torch.bfloat16))


@pytest.mark.parametrize("r", [64, 13, 1])
def test_ragged_multichunk_tsqr(r):
    shapes = [("tall", 5000, 300), ("wide", 200, 4500), ("odd", 2052, 2048)]
    lay = synth.fleet_layout(2, shapes=shapes, r=r, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=7)
    B, A = upload(Bh, Ah)
    mods = api.modules_from_layout(lay)
    F = api.tsqr(mods, B, A)
    assert lf.lf_get_device_status() == 0
    check_tsqr(lay, Bh, Ah, F, range(lay.n))


def test_exact_reconstruction_at_full_rank():
    shapes = [("tall", 5000, 300), ("wide", 200, 4500)]
    lay = synth.fleet_layout(2, shapes=shapes, r=16, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=8)
    B, A = upload(Bh, Ah)
    mods, F, E, st = G.run_factor_path(lay, B, A, lf.policy_U(1, 1))
    assert st == 0
    assert E.ranks.cpu().tolist() == [16] * lay.n
    for i in range(lay.n):
        Bn, An = G.module_np(lay, Bh, Ah, i)
        Bt, Ap = G.exported_module(lay, E, i)
        assert OF.factor_error(Bn, An, Bt, Ap) <= G.RECON_TOL
        np.testing.assert_allclose(Bt @ Bt.T, np.eye(16), atol=1e-4)   # B' orthonormal columns


def test_spectral_policy_ranks_bit_exact_and_errors():
    # one Qwen-like adapter at reduced widths plus a second adapter: S 1/12, floor 1
    shapes = [("q", 896, 896), ("k", 128, 896), ("v", 128, 896), ("o", 896, 896),
              ("gate", 4736, 896), ("up", 4736, 896), ("down", 896, 4736)]
    lay = synth.fleet_layout(2, shapes=shapes, r=64, n_layers=4)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=2)
    B, A = upload(Bh, Ah)
    pol = lf.policy_S(1, 12, 1)
    mods, F, E, st = G.run_factor_path(lay, B, A, pol)
    assert st == 0
    sig = G.oracle_sigma_rows(lay, Bh, Ah, range(lay.n))
    ranks_o, info = OA.spectral_ranks(sig, lay.r, lay.group, 1, 12, 1)
    ranks_g = E.ranks.cpu().numpy()
    assert G.compare_ranks(ranks_g, ranks_o, info, sig, lay.r, lay.group, 1), (ranks_g, ranks_o)
    for g in range(2):
        assert ranks_g[lay.group == g].sum() <= (64 * 28) // 12
    offA = E.off_A.cpu().numpy()
    assert offA[-1] == int((ranks_g.astype(np.int64) * lay.d_in).sum())
    for eg, eo in G.recon_errors(lay, Bh, Ah, E, sig, range(lay.n)):
        assert abs(eg - eo) <= G.RECON_TOL


def test_select_ranks_alone_matches_oracle():
    lay = synth.fleet_layout(6, synth.LLAMA3_8B, r=64)
    sig = synth.sigma_tables(6, synth.LLAMA3_8B, 64, cfg_id=3)
    mods = api.modules_from_layout(lay)
    for pol, (num, den, fl) in ((lf.policy_S(1, 12, 1), (1, 12, 1)), (lf.policy_S(1, 4, 2), (1, 4, 2))):
        ranks, offA, offB = api.select_ranks(mods, pol, torch.from_numpy(sig).cuda())
        assert lf.lf_get_device_status() == 0
        ranks_o, info = OA.spectral_ranks(sig, lay.r, lay.group, num, den, fl)
        assert G.compare_ranks(ranks.cpu().numpy(), ranks_o, info, sig, lay.r, lay.group, fl)
        ro = ranks_o.astype(np.int64)
        assert offA.cpu().numpy().tolist() == [0] + np.cumsum(ro * lay.d_in).tolist()
        assert offB.cpu().numpy().tolist() == [0] + np.cumsum(ro * lay.d_out).tolist()
    ranks, _, _ = api.select_ranks(mods, lf.policy_U(1, 4), torch.from_numpy(sig).cuda())
    assert set(ranks.cpu().tolist()) == {16}


def test_golden_allocation_cases_on_gpu():
    import json, os
    from tests.conftest import GOLDEN
    cases = json.load(open(os.path.join(GOLDEN, "allocation_cases.json")))["spectral"]
    for c in cases:
        n = len(c["r"])
        m = np.zeros(n, dtype=lf.MODULE_DTYPE)
        m["d_out"], m["d_in"], m["r"], m["group"] = 8, 8, c["r"], c["group"]
        sig = np.array(c["sigma"], dtype=np.float64)
        ranks, _, _ = api.select_ranks(m, lf.policy_S(c["num"], c["den"], c["floor"]),
                                       torch.from_numpy(sig).cuda())
        assert ranks.cpu().tolist() == c["ranks"], c["name"]


def test_zero_module_exports_zeros():
    lay = synth.fleet_layout(1, shapes=[("w", 512, 384), ("z", 512, 384)], r=8, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=9)
    b0 = int(lay.B_off[1]); Bh[b0:b0 + 512 * 8] = 0.0
    B, A = upload(Bh, Ah)
    mods, F, E, st = G.run_factor_path(lay, B, A, lf.policy_S(1, 2, 1))
    assert st == 0
    assert F.sigma[1].abs().max().item() == 0.0
    assert int(E.ranks[1]) == 1
    Bt, Ap = G.exported_module(lay, E, 1)
    assert not Bt.any() and not Ap.any()


def test_deterministic_bitwise():
    lay, Bh, Ah = synth.tiny_fleet()
    B, A = upload(Bh, Ah)
    outs = [G.run_factor_path(lay, B, A, lf.policy_S(1, 4)) for _ in range(2)]
    for x, y in ((outs[0][1].R_B, outs[1][1].R_B), (outs[0][1].sigma, outs[1][1].sigma),
                 (outs[0][2].A_pool, outs[1][2].A_pool), (outs[0][2].ranks, outs[1][2].ranks)):
        assert torch.equal(x, y)


def test_pool_capacity_too_small_latches_workspace_error():
    lay, Bh, Ah = synth.tiny_fleet()
    B, A = upload(Bh, Ah)
    mods = api.modules_from_layout(lay)
    F = api.tsqr(mods, B, A)
    pol = lf.policy_U(1, 4)
    E = api.alloc_export(mods, pol, B.device)
    E.A_pool = E.A_pool[:1000]
    api.truncate_export(mods, pol, B, A, F, out=E)
    assert lf.lf_get_device_status() == 4          # LF_ERR_WORKSPACE, latched on the device
    assert lf.lf_get_device_status() == 0          # and cleared by the read


def _planted(d_out, r, sig, seed):
    """B = G diag(sig) H with G (d_out x r) orthonormal and H (r x r) orthogonal: the
    singular values of B are exactly sig (up to fp32 rounding of the stored bytes)."""
    g = np.random.default_rng(seed)
    Gq, _ = np.linalg.qr(g.standard_normal((d_out, r)))
    H, _ = np.linalg.qr(g.standard_normal((r, r)))
    return (Gq * sig) @ H


def test_gram_leaf_accuracy_on_ill_conditioned_factor():
    # cond(B) = 1e3: the fp64 Gram + Cholesky R carries ~1e-16 * cond^2 = 1e-10 relative
    # error before the fp32 store, far inside what fp32 Householder (~u32 * cond) reaches
    r, d_out, d_in = 16, 3000, 700
    lay = synth.fleet_layout(1, shapes=[("m", d_out, d_in)], r=r, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=11)
    b0 = int(lay.B_off[0])
    Bh[b0:b0 + d_out * r] = torch.from_numpy(_planted(d_out, r, np.logspace(0, -3, r), 5).ravel()).float()
    B, A = upload(Bh, Ah)
    mods = api.modules_from_layout(lay)
    F = api.tsqr(mods, B, A)
    assert lf.lf_get_device_status() == 0
    Bn, _ = G.module_np(lay, Bh, Ah, 0)
    want = OF.qr_r(Bn)
    got = F.R_B[0][:r, :r].double().cpu().numpy()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-6


def test_rank_deficient_factors_take_householder_route():
    # a duplicated column, a zero column and cond = 1e7: Cholesky pivots fall below
    # 1e-9 of the Gram diagonal, so these matrices are factored by Householder TSQR;
    # R is then not unique past the rank, but R^T R = X^T X and sigma(B A) are
    r, d_out, d_in = 16, 2500, 2100
    shapes = [("dup", d_out, d_in), ("zero_col", d_out, d_in), ("cond1e7", d_out, d_in), ("ok", d_out, d_in)]
    lay = synth.fleet_layout(1, shapes=shapes, r=r, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=12)
    for i in range(3):
        b0 = int(lay.B_off[i])
        Bm = Bh[b0:b0 + d_out * r].view(d_out, r)
        if i == 0:
            Bm[:, 5] = Bm[:, 2]
        elif i == 1:
            Bm[:, 7] = 0.0
        else:
            Bm[:] = torch.from_numpy(_planted(d_out, r, np.logspace(0, -7, r), 6)).float()
    B, A = upload(Bh, Ah)
    mods = api.modules_from_layout(lay)
    F = api.tsqr(mods, B, A)
    assert lf.lf_get_device_status() == 0
    RB, S = F.R_B.double().cpu().numpy(), F.sigma.cpu().numpy()
    for i in range(lay.n):
        Bn, An = G.module_np(lay, Bh, Ah, i)
        R = RB[i][:r, :r]
        assert np.allclose(np.tril(R, -1), 0) and np.all(np.diag(R) >= 0)
        gram = Bn.T @ Bn
        assert np.linalg.norm(R.T @ R - gram) <= 1e-5 * np.linalg.norm(gram), i
        s, *_ = OF.spectrum_factor(Bn, An)
        assert np.max(np.abs(S[i][:r] - s)) <= G.SIGMA_TOL * s[0], i


@pytest.mark.parametrize("variant", ["absolute_energy", "fleet_global_budget"])
def test_allocation_variants_ranks_bit_exact(variant):
    # allocation variants of the spectral policy: ranking candidates by sigma^2
    # (kind 2), and one budget over every module of the fleet (a single group)
    shapes = [("q", 896, 896), ("k", 128, 896), ("v", 128, 896), ("o", 896, 896),
              ("gate", 4736, 896), ("up", 4736, 896), ("down", 896, 4736)]
    lay = synth.fleet_layout(3, shapes=shapes, r=64, n_layers=2)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=13)
    if variant == "fleet_global_budget":
        lay.group[:] = 0
    B, A = upload(Bh, Ah)
    absolute = variant == "absolute_energy"
    pol = lf.policy_S(1, 12, 1, absolute=absolute)
    mods, F, E, st = G.run_factor_path(lay, B, A, pol)
    assert st == 0
    sig = G.oracle_sigma_rows(lay, Bh, Ah, range(lay.n))
    ranks_o, info = OA.spectral_ranks(sig, lay.r, lay.group, 1, 12, 1, absolute=absolute)
    ranks_g = E.ranks.cpu().numpy()
    assert G.compare_ranks(ranks_g, ranks_o, info, sig, lay.r, lay.group, 1, absolute=absolute), (ranks_g, ranks_o)
    for g in set(lay.group.tolist()):
        assert ranks_g[lay.group == g].sum() <= (64 * int((lay.group == g).sum())) // 12
    for eg, eo in G.recon_errors(lay, Bh, Ah, E, sig, range(lay.n)):
        assert abs(eg - eo) <= G.RECON_TOL


@pytest.mark.parametrize("num,den", [(99, 100), (9, 10), (1, 2)])
def test_energy_fraction_ranks_bit_exact(num, den):
    # kind 3: the smallest rank keeping num/den of each module's spectral energy (the
    # minimal subspace rule of LoRASpace, per module); modules near the threshold are
    # refined in fp64 like the spectral budget's boundary
    shapes = [("q", 896, 896), ("k", 128, 896), ("gate", 4736, 896), ("down", 896, 4736)]
    lay = synth.fleet_layout(3, shapes=shapes, r=64, n_layers=2)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=14)
    B, A = upload(Bh, Ah)
    mods, F, E, st = G.run_factor_path(lay, B, A, lf.policy_E(num, den, 1))
    assert st == 0
    sig = G.oracle_sigma_rows(lay, Bh, Ah, range(lay.n))
    ranks_o, gaps = OA.energy_fraction_ranks(sig, lay.r, num, den, 1)
    ranks_g = E.ranks.cpu().numpy()
    diff = ranks_g != ranks_o
    assert not np.any(diff & (gaps > 1e-12)), (ranks_g[diff], ranks_o[diff], gaps[diff])
    for eg, eo in G.recon_errors(lay, Bh, Ah, E, sig, range(lay.n)):
        assert abs(eg - eo) <= G.RECON_TOL


@pytest.mark.parametrize("r", [64, 36])
def test_integer_leaf_long_rows_and_scale_fallback(r):
    """The integer-Gram leaf takes a matrix in items of at most 24576 rows: a factor of
    26000 rows is two items whose packed Grams are merged in item order.  A factor whose
    first 128 rows are 1e-3 times smaller than the rest exceeds the column scale taken on
    those rows, so the leaf leaves it to the fp64 Gram leaf.  Both must give the oracle's
    R and sigma; the profile shows the integer leaf ran."""
    shapes = [("long", 26000, 400), ("spike", 3000, 512), ("plain", 1000, 26000)]
    lay = synth.fleet_layout(1, shapes=shapes, r=r, n_layers=1)
    Bh = torch.zeros(lay.B_total); Ah = torch.zeros(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=15)
    b0 = int(lay.B_off[1])
    Bh[b0:b0 + 128 * r] *= 1e-3
    B, A = upload(Bh, Ah)
    mods = api.modules_from_layout(lay)
    lf.lf_profile_reset(); lf.lf_profile_enable(True)
    F = api.tsqr(mods, B, A)
    lf.lf_profile_enable(False)
    ph = lf.lf_profile_read()
    assert lf.lf_get_device_status() == 0
    assert ph.get("tsqr_gram_i8", (0, 0))[1] == 1, ph
    check_tsqr(lay, Bh, Ah, F, range(lay.n))
