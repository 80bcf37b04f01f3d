"""Seeded synthetic inputs shaped like the LoRA fleets the LoRAForge pages describe.

This module is the one piece shared by the CUDA path, the tests and the fp64
oracle.  It only draws numbers and lays out buffers; it holds none of the
method's arithmetic (no QR, no SVD, no rank allocation, no LoRA apply).

Shapes
------
* Qwen2.5-7B layer: hidden 3584, kv 512, ffn 18944, 28 layers.
* Llama-3-8B layer: hidden 4096, kv 1024, ffn 14336, 32 layers.
Each layer carries seven adapted projections q, k, v, o, gate, up, down;
module shapes are written (d_out, d_in) as in "Compress then Serve", §3
(B_i is d_B x r_i, A_i is r_i x d_A).

Recipes (all draws are standard normals from a seeded torch or numpy
generator; a per-tensor seed comes from a splitmix64 chain over
(base seed, config id, adapter, module type, tensor id)):
* A  = N(0, 1/d_in) entries, r x d_in, fp32.
* B  = G * diag(sigma): G is a d_out x r Gaussian whose columns are scaled to
  unit length, sigma_j = (j+1)^-1 for the tiny case and
  sigma_j = (j+1)^-1 * exp(0.5 z_j), z_j ~ N(0,1), for the fleets.
* adapter ids: uniform, or Zipf(alpha) over n adapters, i.e. P(i) proportional
  to (i+1)^-alpha on i = 0..n-1, then shuffled.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable

import numpy as np

BASE_SEED = 20261202
MASK64 = (1 << 64) - 1
PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def splitmix64(x: int) -> int:
    """One step of the public splitmix64 mixing function (Steele et al.)."""
    x = (x + 0x9E3779B97F4A7C15) & MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def derive_seed(*key: int) -> int:
    """Fold a tuple of non-negative ints into one 63-bit seed."""
    h = BASE_SEED
    for k in key:
        h = splitmix64(h ^ (int(k) & MASK64))
    return h & ((1 << 63) - 1)


@dataclasses.dataclass(frozen=True)
class ModelShape:
    name: str
    hidden: int
    kv: int
    ffn: int
    layers: int

    def proj_shapes(self):
        """(name, d_out, d_in) for the seven adapted projections of a layer."""
        h, kv, f = self.hidden, self.kv, self.ffn
        return [("q", h, h), ("k", kv, h), ("v", kv, h), ("o", h, h),
                ("gate", f, h), ("up", f, h), ("down", h, f)]


QWEN25_7B = ModelShape("Qwen2.5-7B", 3584, 512, 18944, 28)
LLAMA3_8B = ModelShape("Llama-3-8B", 4096, 1024, 14336, 32)


@dataclasses.dataclass
class FleetLayout:
    """Module descriptors for a fleet, in (adapter, projection, layer) order.

    Arrays are plain numpy (int32/int64) so they can be handed to the C ABI's
    lf_module array without conversion.  Offsets are element offsets into one
    flat fp32 buffer for all B factors and one for all A factors; every offset
    is a multiple of 4 elements (16 bytes).
    """
    d_out: np.ndarray
    d_in: np.ndarray
    r: np.ndarray
    group: np.ndarray
    B_off: np.ndarray
    A_off: np.ndarray
    B_total: int
    A_total: int
    proj: np.ndarray      # projection index 0..6
    layer: np.ndarray

    @property
    def n(self) -> int:
        return int(self.d_out.shape[0])


def _align4(x: int) -> int:
    return (x + 3) // 4 * 4


def fleet_layout(n_adapters: int, model: ModelShape | None = None, r: int = 64,
                 n_layers: int | None = None,
                 shapes: list[tuple[str, int, int]] | None = None) -> FleetLayout:
    """Lay out every (adapter, projection, layer) module of a fleet."""
    if shapes is None:
        shapes = model.proj_shapes()
    L = model.layers if (n_layers is None and model is not None) else (n_layers or 1)
    rows = []
    b_off = a_off = 0
    for a in range(n_adapters):
        for p, (_, d_out, d_in) in enumerate(shapes):
            for l in range(L):
                rows.append((d_out, d_in, r, a, b_off, a_off, p, l))
                b_off += _align4(d_out * r)
                a_off += _align4(r * d_in)
    arr = np.array(rows, dtype=np.int64).reshape(-1, 8)
    return FleetLayout(
        d_out=arr[:, 0].astype(np.int32), d_in=arr[:, 1].astype(np.int32),
        r=arr[:, 2].astype(np.int32), group=arr[:, 3].astype(np.int32),
        B_off=arr[:, 4].copy(), A_off=arr[:, 5].copy(), B_total=b_off, A_total=a_off,
        proj=arr[:, 6].astype(np.int32), layer=arr[:, 7].astype(np.int32))


def sigma_profile(gen_normal, r: int, lognormal: bool):
    """sigma_j = (j+1)^-1, optionally times exp(0.5 z_j)."""
    j = np.arange(1, r + 1, dtype=np.float64)
    s = 1.0 / j
    if lognormal:
        s = s * np.exp(0.5 * gen_normal(r))
    return s


def fill_fleet(layout: FleetLayout, B_buf, A_buf, cfg_id: int, lognormal: bool = True,
               adapters: Iterable[int] | None = None, adapter_base: int = 0):
    """Fill flat fp32 torch buffers (CPU or CUDA) with the fleet's factors.

    Draws are made on the buffers' device with a torch generator seeded per
    (config, adapter, projection); all layers of one projection are drawn in
    one batch.  ``adapter_base`` shifts the adapter id used for seeding so a
    large fleet can be generated chunk by chunk into a buffer that holds a
    few adapters only.
    """
    import torch
    dev = B_buf.device
    n = layout.n
    if adapters is None:
        adapters = sorted(set(int(g) for g in layout.group))
    adapters = list(adapters)
    idx_by_ap: dict[tuple[int, int], list[int]] = {}
    for i in range(n):
        idx_by_ap.setdefault((int(layout.group[i]), int(layout.proj[i])), []).append(i)
    for a in adapters:
        for p in range(7):
            ids = idx_by_ap.get((a, p))
            if not ids:
                continue
            d_out = int(layout.d_out[ids[0]]); d_in = int(layout.d_in[ids[0]])
            r = int(layout.r[ids[0]]); L = len(ids)
            g = torch.Generator(device=dev)
            g.manual_seed(derive_seed(cfg_id, adapter_base + a, p, 0))
            G = torch.randn((L, d_out, r), generator=g, device=dev, dtype=torch.float32)
            G /= torch.linalg.vector_norm(G, dim=1, keepdim=True)
            rng = np.random.Generator(np.random.Philox(derive_seed(cfg_id, adapter_base + a, p, 1)))
            sig = np.stack([sigma_profile(rng.standard_normal, r, lognormal) for _ in range(L)])
            G *= torch.from_numpy(sig.astype(np.float32)).to(dev)[:, None, :]
            A = torch.randn((L, r, d_in), generator=g, device=dev, dtype=torch.float32)
            A *= 1.0 / math.sqrt(d_in)
            # consecutive layers of one projection are laid out back to back
            b0 = int(layout.B_off[ids[0]]); a0 = int(layout.A_off[ids[0]])
            sb = _align4(d_out * r); sa = _align4(r * d_in)
            for t, i in enumerate(ids):
                assert int(layout.B_off[i]) == b0 + t * sb and int(layout.A_off[i]) == a0 + t * sa
            if sb == d_out * r:
                B_buf[b0:b0 + L * sb].view(L, d_out, r).copy_(G)
            else:
                for t in range(L):
                    B_buf[b0 + t * sb:b0 + t * sb + d_out * r].view(d_out, r).copy_(G[t])
            if sa == r * d_in:
                A_buf[a0:a0 + L * sa].view(L, r, d_in).copy_(A)
            else:
                for t in range(L):
                    A_buf[a0 + t * sa:a0 + t * sa + r * d_in].view(r, d_in).copy_(A[t])


def module_view(layout: FleetLayout, B_buf, A_buf, i: int):
    """(B, A) views of module i: B is d_out x r, A is r x d_in."""
    d_out, d_in, r = int(layout.d_out[i]), int(layout.d_in[i]), int(layout.r[i])
    b0, a0 = int(layout.B_off[i]), int(layout.A_off[i])
    return (B_buf[b0:b0 + d_out * r].reshape(d_out, r), A_buf[a0:a0 + r * d_in].reshape(r, d_in))


def tiny_fleet(seed_cfg: int = 0):
    """Tiny case: 4 adapters x one 256x256 module, r=16, sigma_j = 1/j. CPU torch."""
    import torch
    lay = fleet_layout(4, shapes=[("w", 256, 256)], r=16, n_layers=1)
    B = torch.zeros(lay.B_total, dtype=torch.float32)
    A = torch.zeros(lay.A_total, dtype=torch.float32)
    fill_fleet(lay, B, A, cfg_id=seed_cfg, lognormal=False)
    return lay, B, A


def sigma_tables(n_adapters: int, model: ModelShape, r: int, cfg_id: int) -> np.ndarray:
    """Synthetic fp64 singular-value tables, one row of r per module, laid out in
    fleet_layout's (adapter, projection, layer) order: the values
    (j+1)^-1 e^{0.5 z_j}, listed in descending order as singular values are."""
    rows = []
    for a in range(n_adapters):
        rng = np.random.Generator(np.random.Philox(derive_seed(cfg_id, a, 99)))
        for _p in range(7):
            for _l in range(model.layers):
                rows.append(np.sort(sigma_profile(rng.standard_normal, r, True))[::-1])
    return np.ascontiguousarray(np.stack(rows))


def collection_layout(d_out: int, d_in: int, ranks) -> FleetLayout:
    """One module position shared by len(ranks) LoRAs of the given ranks (one group each)."""
    rows = []
    b_off = a_off = 0
    for a, r in enumerate(ranks):
        rows.append((d_out, d_in, int(r), a, b_off, a_off, 0, 0))
        b_off += _align4(d_out * int(r))
        a_off += _align4(int(r) * d_in)
    arr = np.array(rows, dtype=np.int64).reshape(-1, 8)
    return FleetLayout(
        d_out=arr[:, 0].astype(np.int32), d_in=arr[:, 1].astype(np.int32),
        r=arr[:, 2].astype(np.int32), group=arr[:, 3].astype(np.int32),
        B_off=arr[:, 4].copy(), A_off=arr[:, 5].copy(), B_total=b_off, A_total=a_off,
        proj=arr[:, 6].astype(np.int32), layer=arr[:, 7].astype(np.int32))


def fill_collection(layout: FleetLayout, key: tuple[int, ...]):
    """CPU fp32 torch buffers for a collection_layout: B = column-normalised Gaussian
    times sigma_j = (j+1)^-1 e^{0.5 z_j}, A ~ N(0, 1/d_in), seeded per LoRA."""
    import torch
    B = torch.zeros(layout.B_total, dtype=torch.float32)
    A = torch.zeros(layout.A_total, dtype=torch.float32)
    for i in range(layout.n):
        d_out, d_in, r = int(layout.d_out[i]), int(layout.d_in[i]), int(layout.r[i])
        g = torch.Generator()
        g.manual_seed(derive_seed(*key, i, 0))
        Bi = torch.randn((d_out, r), generator=g, dtype=torch.float32)
        Bi /= torch.linalg.vector_norm(Bi, dim=0, keepdim=True)
        rng = np.random.Generator(np.random.Philox(derive_seed(*key, i, 1)))
        Bi *= torch.from_numpy(sigma_profile(rng.standard_normal, r, True).astype(np.float32))[None, :]
        Ai = torch.randn((r, d_in), generator=g, dtype=torch.float32) * (1.0 / math.sqrt(d_in))
        b0, a0 = int(layout.B_off[i]), int(layout.A_off[i])
        B[b0:b0 + d_out * r] = Bi.reshape(-1)
        A[a0:a0 + r * d_in] = Ai.reshape(-1)
    return B, A


def normal_f32(shape, key: tuple[int, ...], device="cpu"):
    """fp32 tensor of N(0, 1) draws (torch, seeded)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(*key))
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def zipf_ids(T: int, n: int, alpha: float, key: tuple[int, ...]) -> np.ndarray:
    """T adapter ids drawn from P(i) ~ (i+1)^-alpha on 0..n-1 (finite support), shuffled."""
    rng = np.random.Generator(np.random.Philox(derive_seed(*key)))
    p = (np.arange(1, n + 1, dtype=np.float64)) ** (-alpha)
    p /= p.sum()
    ids = rng.choice(n, size=T, p=p).astype(np.int32)
    rng.shuffle(ids)
    return ids


def uniform_ids(T: int, n: int, key: tuple[int, ...]) -> np.ndarray:
    rng = np.random.Generator(np.random.Philox(derive_seed(*key)))
    return rng.integers(0, n, size=T, dtype=np.int64).astype(np.int32)


def normal_bf16(shape, key: tuple[int, ...], std: float = 1.0, device="cpu"):
    """bf16 tensor of N(0, std^2) draws (torch, seeded)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(*key))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t *= std
    return t.to(torch.bfloat16)
