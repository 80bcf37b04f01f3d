"""Parity at the benchmark's full sizes, in the launch configuration bench.py times.

* Factor construction fleet: 85 adapters x 196 Qwen2.5-7B-shaped modules, r = 64,
  LoRAForge-S 1/12 floor 1, generated on the GPU.  Rank tables of whole adapters
  (the S budget's scope) must equal the oracle's; sampled modules of every shape are
  checked for R, sigma and reconstruction error.
* Decode apply (Llama-3-8B shapes, T = 256, 128 adapters, Zipf(1) ids) and prefill
  apply (Qwen2.5-7B shapes, 32 x 512 tokens, k = 16 and 64): every token of some
  projections at y0 = 0 (the whole LoRA delta against the oracle) and sampled tokens of
  every projection at the timed y0 ~ N(0, 1), on the same bf16 bytes.
* Large fleet: adapters of the 1024-adapter Llama-3-8B fleet compressed in chunks, then
  the mixed batch (64 prefill segments of 48 tokens + 1024 decode tokens, Zipf(1.2) ids)
  applied through the exported pools; whole-adapter ranks and sampled tokens checked.
"""
import math

import numpy as np
import pytest
import torch

from oracle import allocate as OA
from oracle import apply as OP
from oracle import factor as OF
from post_hoc_rank_b200 import api, build, synth
from post_hoc_rank_b200 import loraforge as lf
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available()


def download_module(lay, B, A, i):
    d_out, d_in, r = int(lay.d_out[i]), int(lay.d_in[i]), int(lay.r[i])
    b0, a0 = int(lay.B_off[i]), int(lay.A_off[i])
    return (B[b0:b0 + d_out * r].view(d_out, r).cpu().numpy(), A[a0:a0 + r * d_in].view(r, d_in).cpu().numpy())


def check_adapter_ranks(lay, B, A, E, adapter, num, den, floor):
    idx = np.nonzero(lay.group == adapter)[0]
    rs = int(lay.r.max())
    sig = np.zeros((len(idx), rs))
    for q, i in enumerate(idx):
        Bm, Am = download_module(lay, B, A, i)
        s, *_ = OF.spectrum_factor(Bm, Am)
        sig[q, :len(s)] = s
    ranks_o, info = OA.spectral_ranks(sig, lay.r[idx], np.zeros(len(idx), int), num, den, floor)
    ranks_g = E.ranks.cpu().numpy()[idx]
    assert G.compare_ranks(ranks_g, ranks_o, info, sig, lay.r[idx], np.zeros(len(idx), int), floor), \
        (adapter, np.nonzero(ranks_g != ranks_o))
    return idx, sig


def test_factor_fleet_full_size():
    dev = torch.device("cuda")
    lay = synth.fleet_layout(85, synth.QWEN25_7B, r=64)
    mods = api.modules_from_layout(lay)
    B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    synth.fill_fleet(lay, B, A, cfg_id=2)
    pol = lf.policy_S(1, 12, 1)
    F = api.tsqr(mods, B, A)
    E = api.truncate_export(mods, pol, B, A, F)
    assert lf.lf_get_device_status() == 0
    ranks = E.ranks.cpu().numpy()
    for g in range(85):
        assert ranks[lay.group == g].sum() <= (196 * 64) // 12
    # whole adapters: first, middle, last
    for adapter in (0, 42, 84):
        idx, sig = check_adapter_ranks(lay, B, A, E, adapter, 1, 12, 1)
        if adapter == 42:
            # every projection shape, two layers each: R, sigma, reconstruction error
            for p in range(7):
                for l in (0, 27):
                    q = p * 28 + l
                    i = int(idx[q])
                    Bm, Am = download_module(lay, B, A, i)
                    r = 64
                    RBo, RAo = OF.qr_r(Bm), OF.qr_r(Am.T)
                    RB = F.R_B[i].cpu().numpy()[:r, :r]; RA = F.R_A[i].cpu().numpy()[:r, :r]
                    assert np.linalg.norm(RB - RBo) <= G.R_TOL * np.linalg.norm(RBo)
                    assert np.linalg.norm(RA - RAo) <= G.R_TOL * np.linalg.norm(RAo)
                    s = sig[q]
                    assert np.abs(F.sigma[i].cpu().numpy() - s).max() <= G.SIGMA_TOL * s[0]
                    Bt, Ap = G.exported_module(lay, E, i)
                    eg = OF.factor_error(Bm, Am, Bt, Ap)
                    assert abs(eg - OF.truncation_error(s, int(ranks[i]))) <= G.RECON_TOL
    del B, A, F, E
    torch.cuda.empty_cache()


def bf16_half_ulp(v):
    """Half a bf16 ulp at |v| (8 significant bits): the error of the one rounding of y."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 8)


def apply_check(x, y0, y, ids, ranks, offA, offB, Ap, Bt, scale, tokens=None):
    """Oracle on the given tokens (all tokens when None), on the same bf16 bytes.

    Element by element, |y - y_oracle| may exceed half a bf16 ulp of y_oracle (the one
    rounding of y = y0 + s B't) by at most APPLY_TOL times the largest LoRA delta
    max|y_oracle - y0| of the checked rows; rows with id -1 must equal y0 bit for bit."""
    ids = np.asarray(ids)
    if tokens is None:
        tokens = np.arange(len(ids))
    xs = x[tokens].float().cpu().numpy()
    ys0 = y0[tokens].float().cpu().numpy()
    ref = OP.lora_apply(xs, ys0, ids[tokens], ranks, offA, offB, Ap.float().cpu().numpy(),
                        Bt.float().cpu().numpy(), scale)
    got = y[tokens].float().cpu().numpy().astype(np.float64)
    err = np.maximum(np.abs(got - ref) - bf16_half_ulp(ref), 0.0).max()
    delta = np.abs(ref - ys0).max()
    assert delta > 0.0
    assert err <= G.APPLY_TOL * delta, (err, delta)
    unrouted = torch.from_numpy(ids < 0)
    assert torch.equal(y[unrouted.to(y.device)], y0[unrouted.to(y.device)])


def make_pools_dev(ranks, d_in, d_out, key, dev):
    rk = np.asarray(ranks, dtype=np.int64)
    offA = np.concatenate([[0], np.cumsum(rk * d_in)]); offB = np.concatenate([[0], np.cumsum(rk * d_out)])
    Ap = synth.normal_bf16((max(int(offA[-1]), 8),), key + (0,), std=d_in ** -0.5, device=dev)
    Bt = synth.normal_bf16((max(int(offB[-1]), 8),), key + (1,), std=d_out ** -0.5, device=dev)
    return offA, offB, Ap, Bt


def run_projection(x, y, ids_d, ranks, offA, offB, Ap, Bt, scale, dev):
    n = len(ranks)
    api.shrink_expand(x, y, ids_d, torch.from_numpy(np.asarray(ranks, np.int32)).to(dev),
                      torch.from_numpy(np.asarray(offA[:-1], np.int64)).to(dev),
                      torch.from_numpy(np.asarray(offB[:-1], np.int64)).to(dev), Ap, Bt, scale)
    assert lf.lf_get_device_status() == 0


def test_decode_full_size_layer():
    dev = torch.device("cuda")
    M = synth.LLAMA3_8B
    n_ad, T = 128, 256
    lay = synth.fleet_layout(n_ad, M, r=64)
    sig = synth.sigma_tables(n_ad, M, 64, cfg_id=3)
    ranks_all, _, _ = api.select_ranks(api.modules_from_layout(lay), lf.policy_S(1, 12, 1),
                                       torch.from_numpy(sig).to(dev))
    ranks_all = ranks_all.cpu().numpy().reshape(n_ad, 7, M.layers)
    ids = synth.zipf_ids(T, n_ad, 1.0, (3, 0))
    ids_d = torch.from_numpy(ids).to(dev)
    g = np.random.default_rng(0)
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        rk = ranks_all[:, p, 0]
        offA, offB, Ap, Bt = make_pools_dev(rk, d_in, d_out, (30, p), dev)
        x = synth.normal_bf16((T, d_in), (31, p), device=dev)
        # every token at y0 = 0 (the check then measures the LoRA delta alone)
        y0 = torch.zeros((T, d_out), dtype=torch.bfloat16, device=dev)
        y = y0.clone()
        run_projection(x, y, ids_d, rk, offA, offB, Ap, Bt, 2.0, dev)
        apply_check(x, y0, y, ids, rk, offA[:-1], offB[:-1], Ap, Bt, 2.0)
        # the timed configuration's y0 ~ N(0, 1), sampled tokens
        y0 = synth.normal_bf16((T, d_out), (32, p), device=dev)
        y = y0.clone()
        run_projection(x, y, ids_d, rk, offA, offB, Ap, Bt, 2.0, dev)
        toks = np.sort(g.choice(T, size=48, replace=False))
        apply_check(x, y0, y, ids, rk, offA[:-1], offB[:-1], Ap, Bt, 2.0, toks)


@pytest.mark.parametrize("k", [16, 64])
def test_prefill_full_size_layer(k):
    dev = torch.device("cuda")
    M = synth.QWEN25_7B
    n_ad, T = 32, 32 * 512
    ids = np.repeat(np.arange(n_ad, dtype=np.int32), 512)
    ids_d = torch.from_numpy(ids).to(dev)
    g = np.random.default_rng(1)
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        rk = [k] * n_ad
        offA, offB, Ap, Bt = make_pools_dev(rk, d_in, d_out, (40, p, k), dev)
        x = synth.normal_bf16((T, d_in), (41, p), device=dev)
        if p in (0, 6):
            # q (3584 -> 3584) and down (18944 -> 3584): every token at y0 = 0
            y0 = torch.zeros((T, d_out), dtype=torch.bfloat16, device=dev)
            y = y0.clone()
            run_projection(x, y, ids_d, rk, offA, offB, Ap, Bt, 2.0, dev)
            apply_check(x, y0, y, ids, rk, offA[:-1], offB[:-1], Ap, Bt, 2.0)
        y0 = synth.normal_bf16((T, d_out), (42, p), device=dev)
        y = y0.clone()
        run_projection(x, y, ids_d, rk, offA, offB, Ap, Bt, 2.0, dev)
        toks = np.sort(g.choice(T, size=24, replace=False))
        apply_check(x, y0, y, ids, rk, offA[:-1], offB[:-1], Ap, Bt, 2.0, toks)


def test_large_fleet_chunked_end_to_end():
    """Adapters 0..63 and 960..1023 of the 1024-adapter Llama fleet (two compression
    chunks), S 1/12 floor 1; then the mixed batch restricted to those adapters."""
    dev = torch.device("cuda")
    M = synth.LLAMA3_8B
    chunk = 64
    exports = {}
    for base in (0, 960):
        lay = synth.fleet_layout(chunk, M, r=64)
        mods = api.modules_from_layout(lay)
        B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
        A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
        synth.fill_fleet(lay, B, A, cfg_id=5, adapter_base=base)
        F = api.tsqr(mods, B, A)
        E = api.truncate_export(mods, lf.policy_S(1, 12, 1), B, A, F)
        assert lf.lf_get_device_status() == 0
        check_adapter_ranks(lay, B, A, E, 0 if base == 0 else chunk - 1, 1, 12, 1)
        exports[base] = (lay, E)
        del B, A, F
        torch.cuda.empty_cache()
    # mixed batch over the 128 resident adapters (ids 0..127 -> fleet adapters 0..63, 960..1023)
    T_pre, seg_len, T_dec = 64 * 48, 48, 1024
    seg_ids = synth.zipf_ids(64, 128, 1.2, (5, 1))
    dec_ids = synth.zipf_ids(T_dec, 128, 1.2, (5, 2))
    ids = np.concatenate([np.repeat(seg_ids, seg_len), dec_ids]).astype(np.int32)
    T = len(ids)
    ids_d = torch.from_numpy(ids).to(dev)
    g = np.random.default_rng(2)
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        # layer 0 module of projection p for every resident adapter, from the bf16 pools
        rk, offA, offB = [], [], []
        pools_A, pools_B = [], []
        baseA = baseB = 0
        for base in (0, 960):
            lay, E = exports[base]
            ranks_e = E.ranks.cpu().numpy()
            offA_e = E.off_A.cpu().numpy(); offB_e = E.off_Bt.cpu().numpy()
            for a in range(chunk):
                i = int(np.nonzero((lay.group == a) & (lay.proj == p) & (lay.layer == 0))[0][0])
                k = int(ranks_e[i])
                rk.append(k)
                pools_A.append(E.A_pool16[int(offA_e[i]):int(offA_e[i]) + k * d_in])
                pools_B.append(E.Bt_pool16[int(offB_e[i]):int(offB_e[i]) + k * d_out])
                offA.append(baseA); offB.append(baseB)
                baseA += k * d_in; baseB += k * d_out
        Ap = torch.cat(pools_A); Bt = torch.cat(pools_B)
        x = synth.normal_bf16((T, d_in), (51, p), device=dev)
        offs = (np.array(offA + [baseA]), np.array(offB + [baseB]))
        if p == 0:
            # every token of the q projection at y0 = 0
            y0 = torch.zeros((T, d_out), dtype=torch.bfloat16, device=dev)
            y = y0.clone()
            run_projection(x, y, ids_d, rk, offs[0], offs[1], Ap, Bt, 2.0, dev)
            apply_check(x, y0, y, ids, rk, np.array(offA), np.array(offB), Ap, Bt, 2.0)
        y0 = synth.normal_bf16((T, d_out), (52, p), device=dev)
        y = y0.clone()
        run_projection(x, y, ids_d, rk, offs[0], offs[1], Ap, Bt, 2.0, dev)
        toks = np.sort(np.concatenate([g.choice(T_pre, 16, replace=False), T_pre + g.choice(T_dec, 16, replace=False)]))
        apply_check(x, y0, y, ids, rk, np.array(offA), np.array(offB), Ap, Bt, 2.0, toks)
