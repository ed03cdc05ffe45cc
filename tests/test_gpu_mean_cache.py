"""Chunked prefill with the block-mean cache (fp2_blockmean_cached /
fp2_prefill_cached): the first chunk of each sequence fills the cache; the
second chunk, attending to the first as a resident prefix, reads the prefix
blocks' means from the cache instead of re-averaging the prefix.  Its block
means and output must be bit-identical to the uncached path, and match the
oracle."""
import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu

B = 128


def chunk_problem(inp, q_rows, lens_q, lens_k, dev="cuda"):
    s = inp.shape
    dtype = fp2.FP2_FP8_E4M3 if s.dtype == "fp8" else fp2.FP2_BF16
    q = torch.cat([inp.q[int(inp.cu_seqlens_q[b]) + a: int(inp.cu_seqlens_q[b]) + e]
                   for b, (a, e) in enumerate(q_rows)]).to(dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32, device=dev)
    lk = torch.tensor(lens_k, dtype=torch.int32, device=dev)
    sc = [x.to(dev) if x is not None else None for x in (inp.q_scale, inp.k_scale, inp.v_scale)]
    return fp2.make_problem(q, inp.k.to(dev), inp.v.to(dev), cu, Hq=s.Hq, Hkv=s.Hkv, d=s.d,
                            block=B, dtype=dtype, max_seqlen_q=max(lens_q),
                            max_seqlen_k=max(lens_k), seqlens_k=lk,
                            page_table=inp.page_table.to(dev), page_size=inp.k.shape[1],
                            q_scale=sc[0], k_scale=sc[1], v_scale=sc[2],
                            out=torch.full((q.shape[0], s.Hq, s.d), float("nan"),
                                           dtype=torch.bfloat16, device=dev))


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_two_chunks_with_mean_cache(dtype):
    prefix = [1024, 512]
    total = [1024 + 700, 512 + 300]
    shape = H.small_shape(total, Hq=8, Hkv=2, dtype=dtype, page_size=64, seed=41)
    inp = synth.make_inputs(shape)
    S, Hkv, d = 2, shape.Hkv, shape.d
    max_blocks = max(-(-L // B) for L in total)
    table = torch.full((S, max_blocks), -1, dtype=torch.int32)
    table[0, :14] = torch.arange(14)
    table[1, :7] = torch.arange(20, 27)
    table = table.cuda()
    num_slots = 32
    cache = torch.full((num_slots, 2, Hkv, d), float("nan"), dtype=torch.float32, device="cuda")

    # chunk 1: the prefixes themselves (no resident keys yet) -> fills the cache
    c1 = chunk_problem(inp, [(0, prefix[0]), (0, prefix[1])], prefix, prefix)
    fp2.prefill_cached(c1.q, c1.k, c1.v, c1.page_table, c1.cu_seqlens, 2.0, B, c1.dtype, c1.out,
                       c1.params, table, max_blocks, cache, num_slots)
    c1.check()
    written = [list(range(8)), list(range(20, 24))]
    for sl in written[0] + written[1]:
        assert torch.isfinite(cache[sl]).all()
    assert torch.isnan(cache[8:14]).all() and torch.isnan(cache[24:27]).all()

    # chunk 2: the new tokens on the resident prefix
    new = [t - p for t, p in zip(total, prefix)]
    rows = [(prefix[0], total[0]), (prefix[1], total[1])]
    orc = []
    for b in range(S):
        Qb = inp.seq_q(b)[prefix[b]:]
        Kb, Vb = inp.seq_k(b), inp.seq_v(b)
        kbar, vbar, cnt = O.blockmean(Kb, Vb, B)
        Sb = O.score(O.pool_q(Qb, B), kbar, prefix[b] // B)
        orc.append((Qb, Kb, Vb, kbar, vbar, cnt, Sb))
    tau = O.tau_for_drop([o[6] for o in orc], [p // B for p in prefix], 0.6, guard=1e-3)

    ref_pr = chunk_problem(inp, rows, new, total)
    ref_pr.prefill(tau)
    ref_pr.check()
    c2 = chunk_problem(inp, rows, new, total)
    fp2.prefill_cached(c2.q, c2.k, c2.v, c2.page_table, c2.cu_seqlens, tau, B, c2.dtype, c2.out,
                       c2.params, table, max_blocks, cache, num_slots)
    c2.check()
    L = c2.layout()
    for name in ("kbar", "vbar"):
        a = c2.ws_view(name, torch.float32, (S, Hkv, L.nkb_max, d))
        e = ref_pr.ws_view(name, torch.float32, (S, Hkv, L.nkb_max, d))
        assert torch.equal(a, e), name
    assert torch.equal(c2.out, ref_pr.out)
    for sl in list(range(14)) + list(range(20, 27)):
        assert torch.isfinite(cache[sl]).all()
    a = 0
    for b in range(S):
        Qb, Kb, Vb, kbar, vbar, cnt, Sb = orc[b]
        keep = O.mask(Sb, prefix[b] // B, tau)
        rws, hds = O.all_rows(Qb.shape[0], Qb.shape[1])
        ref = O.attn_rows(Qb, Kb, Vb, kbar, vbar, cnt, keep, B, rws, hds).reshape(Qb.shape)
        got = c2.out[a: a + new[b]].double().cpu().numpy()
        a += new[b]
        H.assert_close(got, ref, dtype == "fp8", f"seq {b}")


def test_bad_slot_is_reported():
    shape = H.small_shape([300], Hq=8, Hkv=2, page_size=64, seed=43)
    inp = synth.make_inputs(shape)
    pr = H.problem(inp)
    table = torch.tensor([[0, 99, 2]], dtype=torch.int32, device="cuda")
    cache = torch.zeros((4, 2, 2, 128), dtype=torch.float32, device="cuda")
    fp2.blockmean_cached(pr.k, pr.v, pr.page_table, pr.cu_seqlens, table, 3, cache, 4, B,
                         pr.dtype, pr.params)
    st, det = fp2.get_status(pr.params)
    assert st == fp2.FP2_ERR_DEVICE_BOUNDS and det == 4


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_decode_steps_with_mean_cache(dtype):
    """A 1000-token prefill chunk, then three decode steps (one query each).
    Block 7 ends inside the first chunk (1000 = 7*128 + 104), so every step
    re-averages it (it is not wholly inside the step's prefix) and writes it
    back, while blocks 0-6 come from the cache.  Each step must equal the
    uncached call bit for bit and the oracle within tolerance."""
    first, steps = 1000, 3
    total = first + steps
    shape = H.small_shape([total], Hq=8, Hkv=2, dtype=dtype, page_size=64, seed=47)
    inp = synth.make_inputs(shape)
    nblk = -(-total // B)
    table = torch.arange(nblk, dtype=torch.int32).reshape(1, nblk).cuda()
    cache = torch.full((nblk, 2, shape.Hkv, shape.d), float("nan"), dtype=torch.float32,
                       device="cuda")
    c1 = chunk_problem(inp, [(0, first)], [first], [first])
    fp2.prefill_cached(c1.q, c1.k, c1.v, c1.page_table, c1.cu_seqlens, 2.0, B, c1.dtype,
                       c1.out, c1.params, table, nblk, cache, nblk)
    c1.check()
    K, V = inp.seq_k(0), inp.seq_v(0)
    for st in range(steps):
        pos = first + st
        Lk = pos + 1
        kbar, vbar, cnt = O.blockmean(K[:Lk], V[:Lk], B)
        Qd = inp.seq_q(0)[pos:pos + 1]
        Sd = O.score(O.pool_q(Qd, B, pos % B), kbar, pos // B)
        tau = O.tau_for_drop([Sd], [pos // B], 0.5, guard=1e-3)
        keep = O.mask(Sd, pos // B, tau)
        assert keep.sum() < np.isfinite(Sd).sum()  # something is dropped
        ref = O.attn_rows(Qd, K[:Lk], V[:Lk], kbar, vbar, cnt, keep, B,
                          *O.all_rows(1, shape.Hq)).reshape(Qd.shape)
        plain = chunk_problem(inp, [(pos, pos + 1)], [1], [Lk])
        plain.prefill(tau)
        plain.check()
        step = chunk_problem(inp, [(pos, pos + 1)], [1], [Lk])
        fp2.prefill_cached(step.q, step.k, step.v, step.page_table, step.cu_seqlens, tau, B,
                           step.dtype, step.out, step.params, table, nblk, cache, nblk)
        step.check()
        assert torch.equal(step.out, plain.out)
        L = step.layout()
        a = step.ws_view("kbar", torch.float32, (1, shape.Hkv, L.nkb_max, shape.d))
        e = plain.ws_view("kbar", torch.float32, (1, shape.Hkv, L.nkb_max, shape.d))
        assert torch.equal(a, e)
        H.assert_close(step.out.double().cpu().numpy(), ref, dtype == "fp8", f"step {st}")
