"""GPU parity of JD-Full by eigenvalue iteration (lf_jd_full) against the fp64 oracle.

"Compress then Serve" (academ.us/article/2407.00066), §3.1 eq. 1, Appendix 8.1
(case 1) and 8.2.  Both sides start from the same fp32 bases and read the same fp32
factor bytes.

Tolerances.  The GPU forms every contraction in fp64 from fp32 inputs but stores
U_0, V_0, W_i, Z_i, R and the bases in fp32, so each step perturbs the iterate by a
few fp32 ulps times the conditioning of the update (the spread of the top r~
eigenvalues of M, tens here).  The subspaces contract back toward the oracle's; a
rotation inside them does not, so entries of U, V carry the accumulated rounding of
all steps (~1e-5 after ten steps) while the rotation-free quantities stay at the
per-step level:
  * reconstruction U Sigma_i V^T against the oracle's, relative to ||B_i A_i||_F:
    1e-4 (the factor path's tolerance on reconstruction error);
  * objective residual / total: 1e-5 absolute;
  * orthonormality ||U^T U - I||_max, ||V^T V - I||_max: 1e-5 (fp32 storage);
  * entries of U, V: 2e-3 absolute (columns have unit norm).
"""
import numpy as np
import pytest
import torch

from oracle import jd as OJ
from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf

pytestmark = pytest.mark.gpu

REC_TOL = 1e-4
OBJ_TOL = 1e-5
ORTH_TOL = 1e-5
ENTRY_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


class Case:
    """Several problems (module positions), each a collection of LoRAs, in one call."""

    def __init__(self, specs, rank, key):
        self.rank = rank
        mods, Bs, As, positions = [], [], [], []
        boff = aoff = 0
        for p, (d_out, d_in, ranks) in enumerate(specs):
            lay = synth.collection_layout(d_out, d_in, ranks)
            B, A = synth.fill_collection(lay, key + (p,))
            m = api.modules_from_layout(lay)
            m["B_off"] += boff
            m["A_off"] += aoff
            positions.append(list(range(len(mods), len(mods) + lay.n)))
            mods += list(m)
            Bs.append(B)
            As.append(A)
            boff += lay.B_total
            aoff += lay.A_total
        self.mods = np.array(mods, dtype=lf.MODULE_DTYPE)
        self.Bh = torch.cat(Bs)
        self.Ah = torch.cat(As)
        self.tabs = api.jd_tables(self.mods, positions, rank)
        self.positions = positions
        U = torch.zeros(max(self.tabs.U_total, 4), dtype=torch.float32)
        Vt = torch.zeros(max(self.tabs.Vt_total, 4), dtype=torch.float32)
        self.U0, self.V0 = [], []
        for p, pr in enumerate(self.tabs.probs):
            d_out, d_in, uo, vo = int(pr["d_out"]), int(pr["d_in"]), int(pr["U_off"]), int(pr["Vt_off"])
            u = synth.normal_f32((d_out, rank), key + (p, 100))
            v = synth.normal_f32((d_in, rank), key + (p, 101))
            U[uo:uo + d_out * rank] = u.reshape(-1)
            Vt[vo:vo + rank * d_in] = v.t().contiguous().reshape(-1)
            self.U0.append(u.double().numpy())
            self.V0.append(v.double().numpy())
        self.Uh, self.Vth = U, Vt

    def factors(self, p):
        out = []
        for m in self.positions[p]:
            d_out, d_in, r = (int(self.mods[m][k]) for k in ("d_out", "d_in", "r"))
            b0, a0 = int(self.mods[m]["B_off"]), int(self.mods[m]["A_off"])
            out.append((self.Bh[b0:b0 + d_out * r].double().numpy().reshape(d_out, r),
                        self.Ah[a0:a0 + r * d_in].double().numpy().reshape(r, d_in)))
        return [b for b, _ in out], [a for _, a in out]

    def run(self, iters, weights=None, with_sigma=True):
        U, Vt = self.Uh.cuda(), self.Vth.cuda()
        sig = torch.full((max(self.tabs.sigma_total, 1),), float("nan"), device="cuda") if with_sigma else None
        w = torch.tensor(weights, dtype=torch.float64, device="cuda") if weights is not None else None
        api.jd_full(self.mods, self.tabs, self.Bh.cuda(), self.Ah.cuda(), U, Vt, iters, weights=w, sigma=sig)
        st = lf.lf_get_device_status()
        return st, U.cpu(), Vt.cpu(), (sig.cpu() if sig is not None else None)

    def unpack(self, p, U, Vt, sig):
        pr = self.tabs.probs[p]
        d_out, d_in, rt = int(pr["d_out"]), int(pr["d_in"]), self.rank
        uo, vo, so = int(pr["U_off"]), int(pr["Vt_off"]), int(pr["sigma_off"])
        Ug = U[uo:uo + d_out * rt].double().numpy().reshape(d_out, rt)
        Vg = Vt[vo:vo + rt * d_in].double().numpy().reshape(rt, d_in).T
        n = int(pr["count"])
        S = None
        if sig is not None:
            S = [sig[so + j * rt * rt: so + (j + 1) * rt * rt].double().numpy().reshape(rt, rt) for j in range(n)]
        return Ug, Vg, S


def recon_diff(Bs, As, U, V, S, Uo, Vo, So):
    """max_i ||U S_i V^T - Uo So_i Vo^T||_F / ||B_i A_i||_F, in factor space."""
    worst = 0.0
    for B, A, s, so in zip(Bs, As, S, So):
        x2 = np.trace(s.T @ (U.T @ U) @ s @ (V.T @ V))
        y2 = np.trace(so.T @ (Uo.T @ Uo) @ so @ (Vo.T @ Vo))
        xy = np.trace(s.T @ (U.T @ Uo) @ so @ (Vo.T @ V))
        n2 = np.trace((B.T @ B) @ (A @ A.T))
        worst = max(worst, np.sqrt(max(x2 + y2 - 2 * xy, 0.0) / n2))
    return worst


def check(case, iters, weights=None):
    st, U, Vt, sig = case.run(iters, weights)
    assert st == 0, lf.lf_status_string(st)
    g0 = 0
    for p in range(len(case.positions)):
        Bs, As = case.factors(p)
        n = len(Bs)
        w = None if weights is None else weights[g0:g0 + n]
        g0 += n
        Uo, Vo, So = OJ.jd_full(Bs, As, case.U0[p], case.V0[p], iters, weights=w)
        Ug, Vg, Sg = case.unpack(p, U, Vt, sig)
        rt = case.rank
        if iters > 0:
            assert np.max(np.abs(Ug.T @ Ug - np.eye(rt))) <= ORTH_TOL
            assert np.max(np.abs(Vg.T @ Vg - np.eye(rt))) <= ORTH_TOL
        assert np.max(np.abs(Ug - Uo)) <= ENTRY_TOL, (p, np.max(np.abs(Ug - Uo)))
        assert np.max(np.abs(Vg - Vo)) <= ENTRY_TOL, (p, np.max(np.abs(Vg - Vo)))
        assert recon_diff(Bs, As, Ug, Vg, Sg, Uo, Vo, So) <= REC_TOL
        rg, tot = OJ.jd_residual(Bs, As, Ug, Vg, Sg)
        ro, _ = OJ.jd_residual(Bs, As, Uo, Vo, So)
        assert abs(rg - ro) / tot <= OBJ_TOL, (p, rg / tot, ro / tot)
    return U, Vt, sig


def test_two_positions_ten_steps():
    """Two module positions with mixed ranks, the pages' ten iterations."""
    case = Case([(300, 260, [16, 8, 12, 16, 4]), (200, 340, [8, 8, 16])], rank=12, key=(40, 1))
    check(case, 10)


def test_multi_chunk_rows_full_ranks():
    """Rows past one project chunk (2048) with a ragged tail, r = r~ = 64."""
    case = Case([(4100, 2600, [64, 64, 64])], rank=64, key=(40, 2))
    check(case, 3)


def test_unaligned_ranks_and_widths():
    """r_i and r~ not multiples of 4 and d_in not a multiple of 4: element-copy paths."""
    case = Case([(150, 258, [13, 5, 7, 1]), (97, 121, [3, 9])], rank=10, key=(40, 3))
    check(case, 6)


def test_weights_match_oracle():
    case = Case([(180, 160, [8, 8, 8, 8])], rank=6, key=(40, 4))
    check(case, 5, weights=[1.0, 0.25, 4.0, 2.0])


def test_zero_iterations_keep_the_start_and_give_sigma():
    case = Case([(64, 48, [4, 4])], rank=4, key=(40, 5))
    st, U, Vt, sig = case.run(0)
    assert st == 0
    assert torch.equal(U, case.Uh) and torch.equal(Vt, case.Vth)
    Bs, As = case.factors(0)
    Ug, Vg, Sg = case.unpack(0, U, Vt, sig)
    for B, A, S in zip(Bs, As, Sg):
        want = Ug.T @ B @ A @ Vg
        assert np.max(np.abs(S - want)) <= 1e-5 * np.max(np.abs(want))


def test_shared_basis_recovered_exactly():
    """B_i A_i = U* S_i V*^T: the optimum of eq. 1 is zero (closed form)."""
    g = np.random.default_rng(11)
    d_out, d_in, rt, n = 256, 192, 8, 6
    Us = np.linalg.qr(g.standard_normal((d_out, rt)))[0]
    Vs = np.linalg.qr(g.standard_normal((d_in, rt)))[0]
    case = Case([(d_out, d_in, [rt] * n)], rank=rt, key=(40, 6))
    for i, m in enumerate(case.positions[0]):
        b0, a0 = int(case.mods[m]["B_off"]), int(case.mods[m]["A_off"])
        S = g.standard_normal((rt, rt))
        case.Bh[b0:b0 + d_out * rt] = torch.from_numpy((Us @ S).astype(np.float32).reshape(-1))
        case.Ah[a0:a0 + rt * d_in] = torch.from_numpy(Vs.T.astype(np.float32).reshape(-1))
    st, U, Vt, sig = case.run(20)
    assert st == 0
    Bs, As = case.factors(0)
    Ug, Vg, Sg = case.unpack(0, U, Vt, sig)
    res, tot = OJ.jd_residual(Bs, As, Ug, Vg, Sg)
    assert res / tot <= 1e-9
    assert np.max(np.abs(Ug @ Ug.T - Us @ Us.T)) <= 1e-5


def test_deterministic():
    case = Case([(300, 260, [16, 8, 12])], rank=8, key=(40, 7))
    a = case.run(4)
    b = case.run(4)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2]) and torch.equal(a[3], b[3])


def test_rank_deficient_update_reports_numeric():
    """All-zero factors make U_0 = 0: orthogonalize meets R_jj = 0 (LF_ERR_NUMERIC)."""
    case = Case([(64, 48, [4, 4])], rank=4, key=(40, 8))
    case.Bh.zero_()
    st, U, Vt, _ = case.run(1)
    assert st == 5, lf.lf_status_string(st)
    assert torch.isfinite(U).all() and torch.isfinite(Vt).all()
