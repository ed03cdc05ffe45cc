"""Seeded synthetic inputs for block-sparse prefill attention.

This module only draws and lays out inputs: it holds none of the method's
arithmetic, so the CUDA path and the fp64 oracle can both be fed from it.

Recipe (the pages give no dataset for the kernel; these inputs imitate the
shapes the pages benchmark -- 128K-context prefill with GQA, a paged KV cache,
continuous batching and a chunked prefill -- and the block structure that
makes max-based block selection meaningful):

* a latent table ``c ~ N(0, I_d)`` per KV head, so the query heads of one GQA
  group see the same latents;
* every ``B``-token block ``b`` (by absolute position) uses latent ``z(b)``:
  ``z(b) = b`` for the tiny case, else ``z(b) ~ U{0..15}`` drawn once per
  sequence and shared by Q and K, so distant blocks can match;
* ``q = 1.5 c_z + N(0, I)``, ``k = 1.5 c_z + N(0, I)``, the first 4 K rows of
  a sequence times 3 (an attention sink), ``v ~ N(0, I)``;
* draws in fp32 from numpy PCG64 in a fixed order (per sequence: latents,
  latent indices, Q noise, K noise, V), then rounded to bf16 (round to
  nearest even) or quantised to e4m3 with per-head scales absmax/448
  (saturating, round to nearest even);
* paged caches: ``page_size`` tokens per page, pages of every sequence drawn
  from one seeded random permutation of all pages; unused page-table entries
  are -1;
* ``kv_scales="block"`` (e4m3 only): the V rows of key block j of KV head h
  are drawn times 2^(-3 u), u ~ U[0, 1) per (sequence, block, head), so that
  blocks differ in magnitude, and K and V are quantised with one scale per
  (sequence, key block, KV head), absmax/448; each is given as a factor in
  (0, 1] of the per-head reference scale, the largest block scale of the head.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclass
class Shape:
    """One workload: per-sequence query and key lengths and the head layout."""
    lens_q: list
    lens_k: list
    Hq: int
    Hkv: int
    d: int
    B: int
    dtype: str = "bf16"          # "bf16" | "fp8"
    latents: str = "shared16"    # "per_block" | "shared16"
    page_size: int = 0           # 0 = contiguous K/V
    drop: float = 0.8            # target dropped fraction of causal block pairs
    seed: int = 20260822
    kv_scales: str = "head"      # "head" | "block" (e4m3: one K/V scale per key block)


# The five workloads (sizes from the FlashPrefill V2 setting: 128K context on
# a Llama-3-8B-shaped layer, GQA, paged KV, continuous batching, chunked
# prefill at 256K).  seed = 20260822 + workload id.
def workload(cid: int, dtype: str | None = None) -> Shape:
    if cid == 1:
        s = Shape([1024], [1024], 4, 1, 64, 64, "bf16", "per_block", 0, 0.70)
    elif cid == 2:
        s = Shape([32768], [32768], 32, 8, 128, 128, "bf16", "shared16", 0, 0.80)
    elif cid == 3:
        s = Shape([131072], [131072], 32, 8, 128, 128, "bf16", "shared16", 0, 0.80)
    elif cid == 4:
        lens = np.random.Generator(np.random.PCG64(20260822 + 4 + 1000)).integers(
            4096, 65536 + 1, size=8).tolist()
        s = Shape(lens, list(lens), 32, 8, 128, 128, "fp8", "shared16", 64, 0.80)
    elif cid == 5:
        s = Shape([32768], [262144], 64, 8, 128, 128, "fp8", "shared16", 64, 0.85)
    else:
        raise ValueError(f"unknown workload {cid}")
    s.seed = 20260822 + cid
    if dtype is not None:
        s.dtype = dtype
    return s


WORKLOAD_NAMES = {
    1: "tiny causal, 1x1024, Hq4/Hkv1, d64, block64",
    2: "32K causal, Hq32/Hkv8, d128, block128",
    3: "128K causal, Hq32/Hkv8, d128, block128",
    4: "8-seq varlen U[4K,64K], paged 64, Hq32/Hkv8, d128, block128",
    5: "32K chunk on 229376-token paged prefix (256K), Hq64/Hkv8, d128, block128",
}


@dataclass
class Inputs:
    shape: Shape
    q: torch.Tensor                 # [total_q, Hq, d] bf16 | float8_e4m3fn
    k: torch.Tensor                 # [total_k, Hkv, d] or [num_pages, page, Hkv, d]
    v: torch.Tensor
    cu_seqlens_q: torch.Tensor      # int32 [S+1]
    cu_seqlens_k: torch.Tensor      # int32 [S+1] (contiguous offsets)
    seqlens_k: torch.Tensor         # int32 [S]
    page_table: torch.Tensor | None  # int32 [S, max_pages] or None
    q_scale: torch.Tensor | None    # float32 [Hq]
    k_scale: torch.Tensor | None    # float32 [Hkv]
    v_scale: torch.Tensor | None
    _kc: torch.Tensor = field(repr=False, default=None)  # contiguous K (quantised)
    _vc: torch.Tensor = field(repr=False, default=None)
    # per-block scale factors [S, nkb_max, Hkv] (x = e4m3 * scale[h] * factor),
    # or None (one scale per head)
    k_block_factor: torch.Tensor | None = None
    v_block_factor: torch.Tensor | None = None

    @property
    def num_seqs(self) -> int:
        return len(self.shape.lens_q)

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    def _deq(self, x: torch.Tensor, scale: torch.Tensor | None) -> np.ndarray:
        y = x.to(torch.float32).to(torch.float64)
        if scale is not None:
            y = y * scale.to(torch.float64)[None, :, None]
        return y.numpy()

    def seq_q(self, b: int) -> np.ndarray:
        """Dequantised fp64 queries of sequence ``b``: ``[Lq, Hq, d]``."""
        a, e = int(self.cu_seqlens_q[b]), int(self.cu_seqlens_q[b + 1])
        return self._deq(self.q[a:e], self.q_scale)

    def _deq_kv(self, x: torch.Tensor, scale, factor, b: int) -> np.ndarray:
        y = self._deq(x, scale)
        if factor is not None:
            rows = np.arange(y.shape[0]) // self.shape.B  # key block of each row
            y = y * factor[b].to(torch.float64).numpy()[rows][:, :, None]
        return y

    def seq_k(self, b: int) -> np.ndarray:
        a, e = int(self.cu_seqlens_k[b]), int(self.cu_seqlens_k[b + 1])
        return self._deq_kv(self._kc[a:e], self.k_scale, self.k_block_factor, b)

    def seq_v(self, b: int) -> np.ndarray:
        a, e = int(self.cu_seqlens_k[b]), int(self.cu_seqlens_k[b + 1])
        return self._deq_kv(self._vc[a:e], self.v_scale, self.v_block_factor, b)

    def seq_q_rows(self, b: int, rows: np.ndarray) -> np.ndarray:
        a = int(self.cu_seqlens_q[b])
        return self._deq(self.q[a + torch.as_tensor(rows, dtype=torch.long)], self.q_scale)


def _quantise(x: np.ndarray, dtype: str):
    """fp32 [N, H, d] -> (torch tensor in the storage dtype, per-head scale or None)."""
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16), None
    if dtype == "fp8":
        amax = t.abs().amax(dim=(0, 2)).clamp_min(1e-12)
        scale = (amax / E4M3_MAX).to(torch.float32)
        y = (t / scale[None, :, None]).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
        return y, scale
    raise ValueError(dtype)


def _quantise_blocks(parts: list, B: int):
    """Per-block e4m3 quantisation of per-sequence fp32 [L, H, d] arrays:
    (concatenated e4m3 tensor, per-head reference scale [H], factors
    [S, nkb_max, H] in (0, 1]; unused entries 1)."""
    H = parts[0].shape[1]
    nkb = max(-(-p.shape[0] // B) for p in parts)
    bscale = np.ones((len(parts), nkb, H), dtype=np.float64)
    for b, x in enumerate(parts):
        for j in range(-(-x.shape[0] // B)):
            amax = np.abs(x[j * B:(j + 1) * B]).max(axis=(0, 2)).astype(np.float64)
            bscale[b, j] = np.maximum(amax, 1e-12) / E4M3_MAX
    ref = np.zeros(H)
    for b, x in enumerate(parts):
        n = -(-x.shape[0] // B)
        ref = np.maximum(ref, bscale[b, :n].max(axis=0))
    ref32 = ref.astype(np.float32)
    fac = np.ones((len(parts), nkb, H), dtype=np.float32)
    out = []
    for b, x in enumerate(parts):
        n = -(-x.shape[0] // B)
        f = (bscale[b, :n] / ref).astype(np.float32)
        fac[b, :n] = f
        sc = (ref32[None, :] * f)[np.arange(x.shape[0]) // B]  # scale of each row [L, H]
        y = torch.from_numpy(x / sc[:, :, None]).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
        out.append(y)
    return torch.cat(out, dim=0), torch.from_numpy(ref32), torch.from_numpy(fac)


def make_inputs(s: Shape, layout: str | None = None) -> Inputs:
    """Draw the inputs of one workload.  ``layout`` = "contiguous" | "paged" |
    "identity" (a page table whose pages are in order) overrides the shape's
    page size (paged/identity default to 64-token pages)."""
    rng = np.random.Generator(np.random.PCG64(s.seed))
    S = len(s.lens_q)
    Hq, Hkv, d, B = s.Hq, s.Hkv, s.d, s.B
    G = Hq // Hkv
    qs, ks, vs = [], [], []
    for b in range(S):
        Lq, Lk = int(s.lens_q[b]), int(s.lens_k[b])
        P = Lk - Lq
        nblk = -(-Lk // B)
        nlat = nblk if s.latents == "per_block" else 16
        c = rng.standard_normal((Hkv, nlat, d), dtype=np.float32)
        if s.latents == "per_block":
            z = np.arange(nblk)
        else:
            z = rng.integers(0, 16, size=nblk)
        qn = rng.standard_normal((Lq, Hq, d), dtype=np.float32)
        kn = rng.standard_normal((Lk, Hkv, d), dtype=np.float32)
        vv = rng.standard_normal((Lk, Hkv, d), dtype=np.float32)
        zq = z[(P + np.arange(Lq)) // B]                     # latent of each query row
        zk = z[np.arange(Lk) // B]
        head_kv = np.arange(Hq) // G
        # q[t, h] = 1.5 c[h_kv, z(t)] + noise
        qn += 1.5 * c[head_kv[None, :], zq[:, None], :]
        kn += 1.5 * c[np.arange(Hkv)[None, :], zk[:, None], :]
        kn[:4] *= 3.0
        if s.kv_scales == "block":
            vv *= np.exp2(-3.0 * rng.random((nblk, Hkv), dtype=np.float32))[np.arange(Lk) // B][:, :, None]
        qs.append(qn); ks.append(kn); vs.append(vv)
    kfac = vfac = None
    if s.kv_scales == "block":
        if s.dtype != "fp8":
            raise ValueError("per-block scales are an e4m3 input format")
        kc, k_scale, kfac = _quantise_blocks(ks, B)
        vc, v_scale, vfac = _quantise_blocks(vs, B)
        del ks, vs
        qf = np.concatenate(qs, axis=0)
        del qs
        q, q_scale = _quantise(qf, s.dtype); del qf
    else:
        qf = np.concatenate(qs, axis=0)
        kf = np.concatenate(ks, axis=0)
        vf = np.concatenate(vs, axis=0)
        del qs, ks, vs
        q, q_scale = _quantise(qf, s.dtype); del qf
        kc, k_scale = _quantise(kf, s.dtype); del kf
        vc, v_scale = _quantise(vf, s.dtype); del vf
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(s.lens_q)]), dtype=torch.int32)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(s.lens_k)]), dtype=torch.int32)
    seqlens_k = torch.tensor(s.lens_k, dtype=torch.int32)

    layout = layout or ("paged" if s.page_size else "contiguous")
    if layout == "contiguous":
        return Inputs(s, q, kc, vc, cu_q, cu_k, seqlens_k, None, q_scale, k_scale, v_scale,
                      kc, vc, kfac, vfac)
    ps = s.page_size or 64
    npages = [-(-int(L) // ps) for L in s.lens_k]
    total_pages = int(sum(npages))
    if layout == "paged":
        perm = rng.permutation(total_pages).astype(np.int32)
    elif layout == "identity":
        perm = np.arange(total_pages, dtype=np.int32)
    else:
        raise ValueError(layout)
    max_pages = max(npages)
    table = np.full((S, max_pages), -1, dtype=np.int32)
    kcache = torch.zeros((total_pages, ps, Hkv, d), dtype=kc.dtype)
    vcache = torch.zeros((total_pages, ps, Hkv, d), dtype=vc.dtype)
    off = 0
    for b in range(S):
        Lk = int(s.lens_k[b])
        a = int(cu_k[b])
        for p in range(npages[b]):
            phys = int(perm[off + p])
            table[b, p] = phys
            n = min(ps, Lk - p * ps)
            kcache[phys, :n] = kc[a + p * ps: a + p * ps + n]
            vcache[phys, :n] = vc[a + p * ps: a + p * ps + n]
        off += npages[b]
    return Inputs(s, q, kcache, vcache, cu_q, cu_k, seqlens_k, torch.from_numpy(table),
                  q_scale, k_scale, v_scale, kc, vc, kfac, vfac)
