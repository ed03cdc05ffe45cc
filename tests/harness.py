"""Shared test plumbing: move synthetic inputs to the GPU, call the library
through its C ABI, run the fp64 oracle on the same inputs, compare."""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O

BF16_REL_L2, BF16_MAX_ABS = 5e-3, 2e-2
FP8_REL_L2 = 5e-2
NEAR_THRESHOLD = 1e-3


def problem(inp: synth.Inputs, dev: str = "cuda", out_fill: float | None = None,
            ws_fill: int | None = None, group_masks: bool = False,
            attn_kernel: int = 0) -> fp2.Problem:
    s = inp.shape
    dtype = fp2.FP2_FP8_E4M3 if s.dtype == "fp8" else fp2.FP2_BF16
    q = inp.q.to(dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev)
    cu = inp.cu_seqlens_q.to(dev)
    lk = inp.seqlens_k.to(dev)
    pt = inp.page_table.to(dev) if inp.paged else None
    cu_k = None if inp.paged else inp.cu_seqlens_k.to(dev)
    sc = [x.to(dev) if x is not None else None for x in (inp.q_scale, inp.k_scale, inp.v_scale)]
    fac = [x.contiguous().to(dev) if x is not None else None
           for x in (inp.k_block_factor, inp.v_block_factor)]
    out = None
    if out_fill is not None:
        out = torch.full((q.shape[0], s.Hq, s.d), out_fill, dtype=torch.bfloat16, device=dev)
    pr = fp2.make_problem(q, k, v, cu, Hq=s.Hq, Hkv=s.Hkv, d=s.d, block=s.B, dtype=dtype,
                          max_seqlen_q=max(s.lens_q), max_seqlen_k=max(s.lens_k),
                          seqlens_k=lk, cu_seqlens_k=cu_k, page_table=pt,
                          page_size=s.page_size or (k.shape[1] if inp.paged else 0),
                          q_scale=sc[0], k_scale=sc[1], v_scale=sc[2], out=out,
                          group_masks=group_masks, attn_kernel=attn_kernel,
                          k_block_factor=fac[0], v_block_factor=fac[1])
    if ws_fill is not None:
        pr.workspace.fill_(ws_fill)
        fp2.workspace_init(pr.params)
    return pr


def oracle_scores(inp: synth.Inputs):
    """Per sequence: (kbar, vbar, cnt, S, prefix_blocks) from the oracle."""
    res = []
    B = inp.shape.B
    for b in range(inp.num_seqs):
        K, V = inp.seq_k(b), inp.seq_v(b)
        kbar, vbar, cnt = O.blockmean(K, V, B)
        Lq = inp.shape.lens_q[b]
        Lk = inp.shape.lens_k[b]
        pb = (Lk - Lq) // B
        if Lq > 0:
            qbar = pool_q_chunked(inp, b)
            S = O.score(qbar, kbar, pb)
        else:
            S = np.zeros((inp.shape.Hq, 0, kbar.shape[1]))
        res.append((kbar, vbar, cnt, S, pb))
    return res


def pool_q_chunked(inp: synth.Inputs, b: int, chunk_blocks: int = 64):
    """Pooled queries of sequence b, computed block range by block range (so
    a 128K sequence never needs all of Q in fp64 at once).  Query blocks are
    cut at absolute positions: with a prefix P, row t is in block
    (P + t) // B - P // B."""
    B = inp.shape.B
    Lq = inp.shape.lens_q[b]
    off = (inp.shape.lens_k[b] - Lq) % B
    nqb = -(-(off + Lq) // B)
    parts = []
    a = int(inp.cu_seqlens_q[b])
    for i0 in range(0, nqb, chunk_blocks):
        r0 = max(0, i0 * B - off)
        r1 = min(Lq, (i0 + chunk_blocks) * B - off)
        Qc = inp._deq(inp.q[a + r0: a + r1], inp.q_scale)
        parts.append(O.pool_q(Qc, B, off if i0 == 0 else 0))
    return np.concatenate(parts, axis=1)


def pick_tau(orc, drop: float, guard: float = NEAR_THRESHOLD) -> float:
    S_list = [r[3] for r in orc if r[3].shape[1] > 0]
    pb_list = [r[4] for r in orc if r[3].shape[1] > 0]
    return O.tau_for_drop(S_list, pb_list, drop, guard=guard)


def gpu_bits(pr: fp2.Problem, inp: synth.Inputs) -> np.ndarray:
    """Kept mask [S, Hq, nqb_max, nkb_max] (bool) from the workspace bits."""
    L = pr.layout()
    S, Hq = inp.num_seqs, inp.shape.Hq
    w = pr.ws_view("kept_bits", torch.int32, (S, Hq, L.nqb_max, L.nw)).cpu().numpy()
    w = w.view(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(S, Hq, L.nqb_max, L.nw * 32)[..., : L.nkb_max]


def bits_from_keep(keeps, inp: synth.Inputs, L) -> torch.Tensor:
    """Pack per-sequence oracle masks [Hq, nqb, nkb] into the library's
    kept_bits layout [S, Hq, nqb_max, nw] (uint32 stored as int32)."""
    S, Hq = inp.num_seqs, inp.shape.Hq
    full = np.zeros((S, Hq, L.nqb_max, L.nw * 32), dtype=np.uint64)
    for b, keep in enumerate(keeps):
        h, i, j = keep.shape
        full[b, :, :i, :j] = keep
    w = full.reshape(S, Hq, L.nqb_max, L.nw, 32)
    words = (w << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)
    return torch.from_numpy(words.view(np.int32))


def compare(got: np.ndarray, ref: np.ndarray):
    diff = got - ref
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(diff).max()) if diff.size else 0.0
    return rel, mx


def assert_close(got, ref, fp8: bool, what: str = ""):
    rel, mx = compare(got, ref)
    if fp8:
        assert rel <= FP8_REL_L2, f"{what}: rel-L2 {rel:.3e} > {FP8_REL_L2}"
    else:
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, \
            f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"
    return rel, mx


def out_seq(pr: fp2.Problem, inp: synth.Inputs, b: int) -> np.ndarray:
    a, e = int(inp.cu_seqlens_q[b]), int(inp.cu_seqlens_q[b + 1])
    return pr.out[a:e].float().double().cpu().numpy()


def oracle_out(inp: synth.Inputs, b: int, orc_b, keep, rows=None, heads=None):
    kbar, vbar, cnt, S, pb = orc_b
    Q = inp.seq_q(b)
    if rows is None:
        rows, heads = O.all_rows(Q.shape[0], Q.shape[1])
    out = O.attn_rows(Q, inp.seq_k(b), inp.seq_v(b), kbar, vbar, cnt, keep, inp.shape.B,
                      rows, heads)
    return out, rows, heads


def small_shape(lens_q, lens_k=None, Hq=8, Hkv=2, d=128, B=128, dtype="bf16", page_size=0,
                drop=0.7, seed=7, latents="shared16", kv_scales="head") -> synth.Shape:
    lens_k = list(lens_q) if lens_k is None else list(lens_k)
    return synth.Shape(list(lens_q), lens_k, Hq, Hkv, d, B, dtype, latents, page_size, drop, seed,
                       kv_scales)


def drop_fraction(keeps, orc) -> float:
    kept = sum(int(k.sum()) for k in keeps)
    total = 0
    for k, r in zip(keeps, orc):
        Hq, nqb, _ = k.shape
        total += Hq * sum(r[4] + i + 1 for i in range(nqb))
    return 1.0 - kept / max(total, 1)


def finite_tau(t: float) -> float:
    return t if math.isfinite(t) else float("inf")
