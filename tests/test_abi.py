"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, sizes workspaces, and rejects bad arguments on the host
before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

from post_hoc_rank_b200 import build, loraforge as lf, synth
from post_hoc_rank_b200.api import modules_from_layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "loraforge.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lf_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_declared_symbol():
    L = ctypes.CDLL(lf.LIB_PATH)
    syms = header_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(L, s), s
    assert sorted(lf.exported_symbols()) == syms


def test_status_strings():
    for st in range(9):
        assert lf.lf_status_string(st) != "unknown status"


def tiny_mods():
    lay = synth.fleet_layout(4, shapes=[("w", 256, 256)], r=16, n_layers=1)
    return modules_from_layout(lay)


def test_rank_stride_and_workspace_sizes():
    m = tiny_mods()
    assert lf.lf_rank_stride(m) == 16
    assert lf.lf_tsqr_workspace_size(m) > 0
    assert lf.lf_export_workspace_size(m) > 0
    assert lf.lf_select_workspace_size(m) > 0
    assert lf.lf_apply_workspace_size(64, 4) > 0
    assert lf.lf_apply_workspace_size(-1, 4) == 0


def test_pool_bound_uniform_exact_and_spectral_safe():
    m = tiny_mods()
    a, b = lf.lf_export_pool_bound(m, lf.policy_U(1, 4))
    assert (a, b) == (4 * 4 * 256, 4 * 4 * 256)
    # S: 4 groups of one module, r = 16, 1/12 -> K = 1 = floor: only floors
    a, b = lf.lf_export_pool_bound(m, lf.policy_S(1, 12))
    assert (a, b) == (4 * 256, 4 * 256)
    m2 = modules_from_layout(synth.fleet_layout(1, shapes=[("a", 512, 64), ("b", 64, 1024)], r=16, n_layers=1))
    a, b = lf.lf_export_pool_bound(m2, lf.policy_S(1, 2))   # K = 16, extra 14 -> widest module first
    assert a == 1 * 64 + 1 * 1024 + 14 * 1024
    assert b == 1 * 512 + 1 * 64 + 14 * 512


def call_tsqr(m, ws_bytes=1 << 20, **over):
    args = dict(B=16, A=16, RB=16, RA=16, S=16, U=16, V=16)
    args.update(over)
    p, n = m.ctypes.data, m.shape[0]
    return lf.lib().lf_tsqr_batched(p, n, args["B"], args["A"], args["RB"], args["RA"], args["S"],
                                    args["U"], args["V"], 16, ws_bytes, None)


def test_tsqr_rejects_bad_shapes_on_host():
    m = tiny_mods()
    bad = m.copy(); bad["r"][1] = 65
    assert call_tsqr(bad) == 2
    bad = m.copy(); bad["r"][0] = 300
    assert call_tsqr(bad) == 2
    bad = m.copy(); bad["d_in"][2] = 0
    assert call_tsqr(bad) == 2
    bad = m.copy(); bad["A_off"][3] = 6
    assert call_tsqr(bad) == 8
    assert call_tsqr(m, B=0) == 1
    assert call_tsqr(m, A=12) == 8                  # misaligned base pointer
    assert call_tsqr(m, ws_bytes=16) == 4           # workspace too small
    assert lf.lib().lf_tsqr_batched(m.ctypes.data, -1, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert lf.lib().lf_tsqr_batched(m.ctypes.data, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, None) == 0


def test_policy_validation_on_host():
    m = tiny_mods()
    p, n = m.ctypes.data, m.shape[0]
    L = lf.lib()
    bad_policies = [lf.lf_policy(4, 1, 4, 1), lf.lf_policy(-1, 1, 4, 1), lf.lf_policy(0, 1, 0, 1), lf.lf_policy(1, 1, 4, 0),
                    lf.lf_policy(3, 101, 100, 1)]   # kind 3 takes a fraction of the energy (num <= den)
    for pol in bad_policies:
        assert L.lf_select_ranks(p, n, pol, 16, 16, 16, 16, 16, 1 << 20, None) == 1
    assert L.lf_select_ranks(p, n, lf.lf_policy(1, 1, 4, 17), 16, 16, 16, 16, 16, 1 << 20, None) == 2


def test_apply_validation_on_host():
    L = lf.lib()
    ok = dict(T=4, d_in=64, d_out=64, x=16, y=16, ids=16, n=2, ranks=16, oa=16, ob=16, A=16, B=16, ws=16,
              wsb=1 << 20, pa=1024, pb=1024)

    def call(**o):
        a = dict(ok); a.update(o)
        return L.lf_lora_shrink_expand(a["T"], a["d_in"], a["d_out"], a["x"], a["y"], a["ids"], a["n"],
                                       a["ranks"], a["oa"], a["ob"], a["A"], a["B"], a["pa"], a["pb"], 1.0,
                                       None, a["ws"],
                                       a["wsb"], None)
    assert call(T=0) == 0
    assert call(T=-1) == 1
    assert call(d_in=60) == 8
    assert call(d_out=12) == 8
    assert call(x=8) == 8
    assert call(n=0) == 1
    assert call(n=20000) == 1
    assert call(wsb=8) == 4
    assert call(ids=0) == 1
    assert call(pa=-1) == 1


def test_module_dtype_matches_c_struct():
    assert lf.MODULE_DTYPE.itemsize == 32
    assert [lf.MODULE_DTYPE.fields[f][1] for f in ("d_out", "d_in", "r", "group", "B_off", "A_off")] == \
        [0, 4, 8, 12, 16, 24]


def test_jd_problem_dtype_matches_c_struct():
    assert lf.JD_PROBLEM_DTYPE.itemsize == 48
    assert [lf.JD_PROBLEM_DTYPE.fields[f][1] for f in
            ("d_out", "d_in", "rank", "first", "count", "U_off", "Vt_off", "sigma_off")] == \
        [0, 4, 8, 12, 16, 24, 32, 40]


def test_jd_validation_on_host():
    """lf_jd_full rejects bad problem tables before any CUDA call."""
    from post_hoc_rank_b200 import api
    lay = synth.collection_layout(40, 36, [4, 4, 3])
    mods = modules_from_layout(lay)
    tabs = api.jd_tables(mods, [[0, 1, 2]], 4)
    assert lf.lf_jd_workspace_size(mods, tabs.members, tabs.probs) > 0

    def call(members=None, probs=None, iters=1, ptr=16, ws=16, wsb=1 << 24):
        members = tabs.members if members is None else members
        probs = tabs.probs.copy() if probs is None else probs
        return lf.lib().lf_jd_full(
            mods.ctypes.data, len(mods), members.ctypes.data, len(members), probs.ctypes.data, len(probs),
            ptr, ptr, None, iters, ptr, ptr, None, ws, wsb, None)

    def with_prob(**kv):
        p = tabs.probs.copy()
        for k, v in kv.items():
            p[0][k] = v
        return p
    assert call(iters=-1) == 1
    assert call(probs=with_prob(rank=0)) == 2
    assert call(probs=with_prob(rank=65)) == 2
    assert call(probs=with_prob(rank=37)) == 2            # > d_in
    assert call(probs=with_prob(count=0)) == 1
    assert call(probs=with_prob(count=4)) == 1            # past the member list
    assert call(probs=with_prob(d_out=41)) == 2           # members of another shape
    assert call(probs=with_prob(U_off=2)) == 8
    assert call(members=np.array([0, 1, 7], dtype=np.int32)) == 1
    assert call(ptr=0) == 1
    assert call(ptr=8) == 8
    assert call(wsb=64) == 4
    assert call(probs=tabs.probs[:0]) == 0                # nothing to do


def test_route_tokens_validation_on_host():
    L = lf.lib()
    assert L.lf_route_tokens(0, None, 4, None, 0, None) == 0          # empty batch: nothing to do
    assert L.lf_route_tokens(-1, 16, 4, 16, 1 << 20, None) == 1
    assert L.lf_route_tokens(8, 16, 0, 16, 1 << 20, None) == 1
    assert L.lf_route_tokens(8, None, 4, 16, 1 << 20, None) == 1
    assert L.lf_route_tokens(1000, 16, 4, 16, 64, None) == 4          # workspace too small


def test_routed_apply_validation_on_host():
    """The routed entry point applies the same host checks as the unrouted one."""
    L = lf.lib()
    sl = (lf.lf_slice * 1)(lf.lf_slice(64, 0, 0, 16, 16, 16, 16, 16, 1024, 1024))

    def call(T=4, d_in=64, ns=1, x=16, ws=16, wsb=1 << 20, y_ld=64):
        return L.lf_lora_shrink_expand_slices_routed(T, d_in, x, 16, y_ld, 16, 2, sl, ns, 1.0, None, ws, wsb, None)
    assert call(T=0) == 0
    assert call(T=-1) == 1
    assert call(ns=0) == 1
    assert call(ns=5) == 1
    assert call(d_in=60) == 8
    assert call(x=8) == 8
    assert call(wsb=8) == 4
    assert call(ws=None) == 1


def test_pool_module_host_checks():
    """The stacked-row module of a pool (LoRASpace pool subspace): one module whose A is
    the back-to-back stack and whose B is the identity of the summed rank; rejected on
    the host when the factors are not contiguous or the summed rank exceeds 64 or d_in."""
    from post_hoc_rank_b200 import api
    m = api.pool_module([100, 100 + 16 * 256, 100 + 24 * 256], [16, 8, 12], 256)
    assert m.shape == (1,)
    assert (int(m["d_out"][0]), int(m["d_in"][0]), int(m["r"][0]), int(m["A_off"][0]), int(m["B_off"][0])) == (36, 256, 36, 100, 0)
    for bad in [([0, 5], [4, 4], 256), ([0, 40 * 256], [40, 40], 256), ([0], [300], 1024), ([0], [8], 4), ([0, 8], [4], 2), ([], [], 8)]:
        with pytest.raises(ValueError):
            api.pool_module(*bad)


def test_bounded_wait_check_rejects_bad_poll_counts():
    L = lf.lib()
    assert L.lf_check_bounded_wait(-1, None) == 1          # LF_ERR_INVALID_ARG, nothing launched
    assert L.lf_check_bounded_wait((1 << 20) + 1, None) == 1


def test_slice_rank_bound_validation_on_host():
    """lf_slice.max_rank: 0 (no bound) or 1..64; anything else is rejected before a launch."""
    L = lf.lib()
    for bound in (-1, 65, 1000):
        sl = (lf.lf_slice * 1)(lf.lf_slice(64, bound, 0, 16, 16, 16, 16, 16, 1024, 1024))
        assert L.lf_lora_shrink_expand_slices(4, 64, 16, 16, 64, 16, 2, sl, 1, 1.0, None, None, 16, 1 << 20,
                                              None) == 1


def test_projections_validation_on_host():
    """lf_lora_shrink_expand_projections: host checks per projection, before any launch."""
    L = lf.lib()

    def proj(x=16, y=16, d_in=64, reserved=0, y_ld=64, bound=0):
        return lf.lf_projection(x, y, d_in, reserved, y_ld, lf.lf_slice(64, bound, 0, 16, 16, 16, 16, 16, 1024, 1024))

    def call(projs, T=4, ids=16, n=2):
        arr = (lf.lf_projection * max(1, len(projs)))(*projs)
        return L.lf_lora_shrink_expand_projections(T, ids, n, arr, len(projs), 1.0, None, None, 0, None)
    assert lf.MAX_PROJECTIONS == 8
    assert call([proj()], T=0) == 0                      # empty batch: nothing to do
    assert call([]) == 1
    assert call([proj()] * 9) == 1                       # more than LF_MAX_PROJECTIONS
    assert call([proj()], T=-1) == 1
    assert call([proj()], ids=None) == 1
    assert call([proj(), proj(reserved=1)]) == 1
    assert call([proj(), proj(bound=65)]) == 1
    assert call([proj(x=18)]) == 8                       # x not 16-byte aligned
    assert call([proj(d_in=60)]) == 8                    # d_in not a multiple of 8
    assert call([proj(y_ld=48)]) == 1                    # the slice does not fit in y's row
    assert call([proj(x=None)]) == 1
