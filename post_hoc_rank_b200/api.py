"""Convenience layer over the C ABI: allocates outputs/workspaces as torch CUDA
tensors and calls the binding.  No arithmetic of the method happens here."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import loraforge as lf


def modules_from_layout(layout) -> np.ndarray:
    """lf_module array from a synth.FleetLayout (or any object with the same fields)."""
    m = np.zeros(layout.n, dtype=lf.MODULE_DTYPE)
    m["d_out"], m["d_in"], m["r"], m["group"] = layout.d_out, layout.d_in, layout.r, layout.group
    m["B_off"], m["A_off"] = layout.B_off, layout.A_off
    return m


@dataclasses.dataclass
class Factors:
    R_B: torch.Tensor
    R_A: torch.Tensor
    sigma: torch.Tensor
    U: torch.Tensor
    V: torch.Tensor
    rs: int


@dataclasses.dataclass
class Export:
    ranks: torch.Tensor
    off_A: torch.Tensor
    off_Bt: torch.Tensor
    A_pool: torch.Tensor
    Bt_pool: torch.Tensor
    A_pool16: torch.Tensor | None
    Bt_pool16: torch.Tensor | None


def workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def alloc_factors(mods: np.ndarray, device) -> Factors:
    n = mods.shape[0]
    rs = lf.lf_rank_stride(mods)
    f32 = dict(dtype=torch.float32, device=device)
    f64 = dict(dtype=torch.float64, device=device)
    return Factors(torch.empty((n, rs, rs), **f32), torch.empty((n, rs, rs), **f32),
                   torch.empty((n, rs), **f64), torch.empty((n, rs, rs), **f64),
                   torch.empty((n, rs, rs), **f64), rs)


def tsqr(mods, B_base, A_base, out: Factors | None = None, ws=None, stream=None) -> Factors:
    dev = B_base.device
    out = out or alloc_factors(mods, dev)
    ws = ws if ws is not None else workspace(lf.lf_tsqr_workspace_size(mods), dev)
    lf.lf_tsqr_batched(mods, B_base, A_base, out.R_B, out.R_A, out.sigma, out.U, out.V, ws, stream)
    return out


def alloc_export(mods, pol, device, bf16: bool = True) -> Export:
    n = mods.shape[0]
    capA, capB = lf.lf_export_pool_bound(mods, pol)
    i64 = dict(dtype=torch.int64, device=device)
    return Export(torch.empty(n, dtype=torch.int32, device=device), torch.empty(n + 1, **i64),
                  torch.empty(n + 1, **i64),
                  torch.empty(max(capA, 8), dtype=torch.float32, device=device),
                  torch.empty(max(capB, 8), dtype=torch.float32, device=device),
                  torch.empty(max(capA, 8), dtype=torch.bfloat16, device=device) if bf16 else None,
                  torch.empty(max(capB, 8), dtype=torch.bfloat16, device=device) if bf16 else None)


def truncate_export(mods, pol, B_base, A_base, F: Factors, out: Export | None = None, ws=None,
                    stream=None, bf16: bool = True) -> Export:
    dev = B_base.device
    out = out or alloc_export(mods, pol, dev, bf16)
    ws = ws if ws is not None else workspace(lf.lf_export_workspace_size(mods), dev)
    lf.lf_truncate_export(mods, pol, B_base, A_base, F.R_B, F.R_A, F.sigma, F.U, F.V, out.ranks,
                          out.off_A, out.off_Bt, out.A_pool, out.Bt_pool, out.A_pool16, out.Bt_pool16,
                          ws, stream)
    return out


def select_ranks(mods, pol, sigma, stream=None):
    dev = sigma.device
    n = mods.shape[0]
    ranks = torch.empty(n, dtype=torch.int32, device=dev)
    offA = torch.empty(n + 1, dtype=torch.int64, device=dev)
    offB = torch.empty(n + 1, dtype=torch.int64, device=dev)
    ws = workspace(lf.lf_select_workspace_size(mods), dev)
    lf.lf_select_ranks(mods, pol, sigma, ranks, offA, offB, ws, stream)
    return ranks, offA, offB


def pool_module(A_offs, ranks, d_in: int) -> np.ndarray:
    """lf_module of a pool's stacked row factors (LoRASpace's pool-wide subspace, the
    arXiv listing abstract): the A_i (r_i x d_in) of one module position stored back to
    back from element A_offs[0] of a pool form one contiguous (sum r_i) x d_in matrix,
    entered as the A factor of one module whose B factor is the identity of order
    sum r_i, so the module's singular values are those of the stack.  Host checks only:
    sum r_i <= 64 (the kernels' rank limit) and <= d_in, and the factors contiguous."""
    A_offs = [int(o) for o in A_offs]
    ranks = [int(r) for r in ranks]
    if not ranks or len(A_offs) != len(ranks) or min(ranks) < 1:
        raise ValueError("one offset and a positive rank per LoRA")
    R = sum(ranks)
    if R > 64 or R > d_in:
        raise ValueError("the stacked rank must be at most 64 and at most d_in")
    for i in range(len(ranks) - 1):
        if A_offs[i + 1] != A_offs[i] + ranks[i] * d_in:
            raise ValueError("the pool's row factors must be stored back to back")
    m = np.zeros(1, dtype=lf.MODULE_DTYPE)
    m["d_out"], m["d_in"], m["r"], m["group"], m["B_off"], m["A_off"] = R, d_in, R, 0, 0, A_offs[0]
    return m


def pool_subspace_rows(A_base, A_offs, ranks, d_in: int, num: int = 99, den: int = 100, stream=None):
    """Pool-wide subspace of stacked row factors on the GPU: lf_tsqr_batched on
    pool_module (singular values of the stack), then lf_select_ranks with the
    energy-fraction policy (floor 1).  Returns (k, sigma[sum r_i] fp64, Factors)."""
    mods = pool_module(A_offs, ranks, d_in)
    R = int(mods["r"][0])
    eye = torch.eye(R, dtype=torch.float32, device=A_base.device)
    F = tsqr(mods, eye.reshape(-1), A_base, stream=stream)
    k, _, _ = select_ranks(mods, lf.policy_E(num, den, 1), F.sigma, stream=stream)
    return int(k[0].item()), F.sigma[0, :R], F


@dataclasses.dataclass
class PoolSubspace:
    k: torch.Tensor        # int32 [1]
    sigma: torch.Tensor    # fp64 [R], descending
    basis: torch.Tensor    # fp32 [R, d], row j = direction j
    coef: torch.Tensor     # fp32 [R, R], coef[a, j] = stack vector a . direction j
    resid: torch.Tensor    # fp64 [1]


def pool_subspace(base, offs, ranks, d: int, side: str = "row", num: int = 99, den: int = 100, stream=None):
    """LoRASpace's pool-wide subspace of a pool's stacked factors on the GPU
    (lf_pool_subspace): side "row" stacks the A_i (r_i x d) stored at element offsets
    offs of `base`, side "col" puts the B_i (d x r_i) side by side.  Allocates the
    outputs and the workspace as torch tensors."""
    sd = {"row": 0, "col": 1}[side]
    R = int(sum(int(r) for r in ranks))
    dev = base.device
    ws = workspace(lf.lf_pool_workspace_size(sd, ranks, offs, d), dev)
    out = PoolSubspace(torch.zeros(1, dtype=torch.int32, device=dev), torch.zeros(R, dtype=torch.float64, device=dev),
                       torch.zeros(R, d, dtype=torch.float32, device=dev),
                       torch.zeros(R, R, dtype=torch.float32, device=dev),
                       torch.zeros(1, dtype=torch.float64, device=dev))
    lf.lf_pool_subspace(sd, ranks, offs, d, base, num, den, out.k, out.sigma, out.basis, out.coef, out.resid, ws,
                        stream)
    return out


def shrink_expand(x, y, ids, ranks, off_A, off_Bt, A_pool, Bt_pool, scale, ws=None, seg_out=None,
                  stream=None):
    n_adapters = ranks.numel()
    ws = ws if ws is not None else workspace(lf.lf_apply_workspace_size(x.shape[0], n_adapters), x.device)
    lf.lf_lora_shrink_expand(x, y, ids, n_adapters, ranks, off_A, off_Bt, A_pool, Bt_pool, scale, ws,
                             seg_out, stream)
    return y


def shrink_expand_slices(x, y, ids, slices, scale, adapter_scale=None, ws=None, seg_out=None, stream=None):
    """Side path of several output slices sharing x.  slices: list of tuples
    (d_out, y_offset, ranks, off_A, off_Bt, A_pool, Bt_pool) with device tensors
    (ranks int32 and offsets int64 per adapter, bf16 pools); y is T x y_ld."""
    n_adapters = slices[0][2].numel()
    ns = len(slices)
    ws = ws if ws is not None else workspace(lf.lf_apply_slices_workspace_size(x.shape[0], n_adapters, ns), x.device)
    sl = [lf.make_slice(*t) for t in slices]
    lf.lf_lora_shrink_expand_slices(x, y, ids, n_adapters, sl, scale, ws, adapter_scale, seg_out, stream)
    return y


@dataclasses.dataclass
class JdTables:
    members: np.ndarray    # int32 module indices, problem by problem
    probs: np.ndarray      # lf_jd_problem records
    U_total: int           # fp32 elements of the U buffer
    Vt_total: int          # fp32 elements of the V^T buffer
    sigma_total: int       # fp32 elements of the Sigma buffer


def jd_tables(mods: np.ndarray, positions, rank: int) -> JdTables:
    """Problem table for JD-Full over module positions.  positions: one list of module
    indices per problem (the LoRAs sharing that position, all of one shape).  U, V^T and
    Sigma of consecutive problems are laid out back to back (offsets multiples of 4)."""
    members, rows = [], []
    u = v = sg = 0
    for pos in positions:
        pos = [int(m) for m in pos]
        d_out, d_in = int(mods["d_out"][pos[0]]), int(mods["d_in"][pos[0]])
        rows.append((d_out, d_in, rank, len(members), len(pos), u, v, sg))
        members += pos
        u += (d_out * rank + 3) // 4 * 4
        v += (rank * d_in + 3) // 4 * 4
        sg += len(pos) * rank * rank
    probs = np.zeros(len(rows), dtype=lf.JD_PROBLEM_DTYPE)
    for i, r in enumerate(rows):
        probs[i] = r
    return JdTables(np.asarray(members, dtype=np.int32), probs, u, v, sg)


def jd_full(mods, tabs: JdTables, B_base, A_base, U, Vt, iters: int, weights=None, sigma=None, ws=None,
            stream=None):
    """JD-Full eigenvalue iteration in place on U / Vt (fp32 device buffers laid out by
    jd_tables); writes Sigma_i into `sigma` when given."""
    ws = ws if ws is not None else workspace(lf.lf_jd_workspace_size(mods, tabs.members, tabs.probs), U.device)
    lf.lf_jd_full(mods, tabs.members, tabs.probs, B_base, A_base, weights, iters, U, Vt, sigma, ws, stream)
    return U, Vt, sigma


def device_status(stream=None) -> int:
    return lf.lf_get_device_status(stream)
