"""Parity at the full workload sizes, in the launch configuration the bench
times (fp2_prefill over the whole layer).

The oracle computes every block mean, pooled score and mask of the layer.
tau is the plain midpoint rule at the target drop, so some scores lie within
1e-3 of the threshold, where the GPU's fp32 scores may decide either way:
  * the GPU's mask must equal the oracle's everywhere except those pairs;
  * fp2_attn run on the ORACLE's mask is compared with the oracle's output;
  * fp2_prefill (the GPU's own mask) is compared on every row of the checked
    blocks: heads whose GPU mask row equals the oracle's against the same
    oracle output, heads whose mask row differs (near-threshold pairs only)
    against the oracle re-run on the GPU's mask row.
Which rows are checked: the 32K layer every row of every head; the other
workloads 32 query blocks spread over the sequences (each sequence's last
block included), 8 heads each, rotating so that the blocks together cover
every head.
"""
import numpy as np
import pytest

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu

# (workload, dtype, sampled query blocks; None = every block and head)
WORKLOADS = [(3, "bf16", 32), (3, "fp8", 32), (2, "bf16", None), (4, "fp8", 32), (5, "fp8", 32)]


def _samples(orc, n_sample, Hq):
    """[(b, i, heads)] of the blocks to check."""
    nqb = [r[3].shape[1] for r in orc]
    if n_sample is None:
        allh = np.arange(Hq, dtype=np.int32)
        return [(b, i, allh) for b in range(len(orc)) for i in range(nqb[b])]
    rng = np.random.default_rng(4242)
    total = sum(nqb)
    picks = []
    for b, n in enumerate(nqb):
        if n == 0:
            continue
        m = max(1, round(n_sample * n / total))
        blocks = {n - 1} | set(rng.choice(n, size=min(n, m), replace=False).tolist())
        picks += [(b, int(i)) for i in sorted(blocks)]
    stride = max(1, Hq // 8)
    out = []
    for k, (b, i) in enumerate(picks):
        heads = (np.arange(0, Hq, stride, dtype=np.int32) + k % stride) % Hq
        out.append((b, i, heads))
    return out


@pytest.mark.parametrize("cid,dtype,n_sample", WORKLOADS,
                         ids=[f"w{c}-{d}" for c, d, _ in WORKLOADS])
def test_full_size(cid, dtype, n_sample):
    shape = synth.workload(cid, dtype)
    inp = synth.make_inputs(shape)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, shape.drop, guard=0.0)
    fp8 = dtype == "fp8"
    B = shape.B
    pr = H.problem(inp, out_fill=float("nan"))
    pr.prefill(tau)
    pr.check()
    got_bits = H.gpu_bits(pr, inp)
    keeps = []
    near_total = kept_total = causal_total = 0
    for b, (kbar, vbar, cnt, S, pb) in enumerate(orc):
        keep = O.mask(S, pb, tau)
        keeps.append(keep)
        Hq, nqb, nkb = S.shape
        for i in range(nqb):
            iabs = pb + i
            row = S[:, i, : iabs + 1]
            m = row.max(axis=1, keepdims=True)
            near = np.abs(row - (m - tau)) < H.NEAR_THRESHOLD
            agree = got_bits[b, :, i, : iabs + 1] == keep[:, i, : iabs + 1].astype(bool)
            assert (agree | near).all(), f"seq {b} block {i}: mask differs away from threshold"
            near_total += int(near.sum())
            kept_total += int(keep[:, i].sum())
            causal_total += Hq * (iabs + 1)
            assert not got_bits[b, :, i, iabs + 1:].any()
    drop = 1.0 - kept_total / causal_total
    assert abs(drop - shape.drop) < 0.01, drop
    out_prefill = pr.out.clone()
    # fp2_attn on the oracle's mask
    bits = H.bits_from_keep(keeps, inp, pr.layout()).cuda()
    pr.out.fill_(float("nan"))
    fp2.attn(pr.q, pr.k, pr.v, pr.page_table, pr.cu_seqlens, bits, B, pr.dtype, pr.out,
             pr.params)
    pr.check()
    rows = rows_own_mask = rows_gpu_mask = 0
    cache = {}
    for b, i, heads in _samples(orc, n_sample, shape.Hq):
        if b not in cache:
            cache.clear()
            cache[b] = (inp.seq_k(b), inp.seq_v(b))
        K, V = cache[b]
        kbar, vbar, cnt, S, pb = orc[b]
        off = (shape.lens_k[b] - shape.lens_q[b]) % B
        r0, r1 = max(0, i * B - off), min(shape.lens_q[b], (i + 1) * B - off)
        a = int(inp.cu_seqlens_q[b])
        Qb = inp._deq(inp.q[a + r0: a + r1], inp.q_scale)
        p0 = pb * B + off + r0
        iabs = pb + i
        ref = O.attn_query_block(Qb, K, V, kbar, vbar, cnt, keeps[b][:, i], B, iabs, heads,
                                 p0=p0).reshape(r1 - r0, heads.size, -1)
        got = pr.out[a + r0: a + r1].double().cpu().numpy()[:, heads]
        H.assert_close(got, ref, fp8, f"w{cid} seq {b} block {i} (fp2_attn, oracle mask)")
        # fp2_prefill: every row, each head against the oracle on the mask row
        # the GPU took for it
        gpu_row = got_bits[b, :, i, : keeps[b].shape[2]].astype(np.uint8)
        differs = (gpu_row[heads, : iabs + 1] != keeps[b][heads, i, : iabs + 1]).any(axis=1)
        want = ref.copy()
        if differs.any():
            dh = heads[differs]
            keep_gpu = keeps[b][:, i].copy()
            keep_gpu[dh] = gpu_row[dh]
            want[:, differs] = O.attn_query_block(Qb, K, V, kbar, vbar, cnt, keep_gpu, B, iabs,
                                                  dh, p0=p0).reshape(r1 - r0, dh.size, -1)
        gp = out_prefill[a + r0: a + r1].double().cpu().numpy()[:, heads]
        H.assert_close(gp, want, fp8, f"w{cid} seq {b} block {i} (fp2_prefill, own mask)")
        rows += (r1 - r0) * heads.size
        rows_gpu_mask += (r1 - r0) * int(differs.sum())
        rows_own_mask += (r1 - r0) * int((~differs).sum())
    assert rows > 0 and rows == rows_own_mask + rows_gpu_mask
    if n_sample is None:
        assert rows == sum(shape.lens_q) * shape.Hq
    print(f"w{cid}-{dtype}: tau={tau:.4f} drop={drop:.4f} near-threshold pairs={near_total} "
          f"rows compared={rows} (on the GPU's differing mask: {rows_gpu_mask})")


# dense runs (every block kept), as the bench times them for its own-dense
# baseline: too long for the per-row oracle, so query blocks are sampled and
# the keep-all special case is checked against dense causal attention
DENSE = [(3, "bf16"), (3, "fp8")]
DENSE_BLOCKS = 64


@pytest.mark.parametrize("cid,dtype", DENSE, ids=[f"w{c}-{d}-dense" for c, d in DENSE])
def test_full_size_dense(cid, dtype):
    """tau = +inf at full size: the GPU mask keeps every causal block and the
    output equals dense causal attention, on 64 seeded query blocks of every
    sequence's blocks (the last one included), every head of each."""
    import concurrent.futures as cf
    import math
    import os
    shape = synth.workload(cid, dtype)
    inp = synth.make_inputs(shape)
    fp8 = dtype == "fp8"
    B = shape.B
    pr = H.problem(inp, out_fill=float("nan"))
    pr.prefill(math.inf)
    pr.check()
    got_bits = H.gpu_bits(pr, inp)
    rng = np.random.default_rng(777)
    rows = 0
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        for b in range(inp.num_seqs):
            Lq, Lk = shape.lens_q[b], shape.lens_k[b]
            P = Lk - Lq
            pb, off = P // B, P % B
            nqb = -(-(off + Lq) // B)
            # every causal block kept, nothing past the diagonal
            for i in range(nqb):
                assert got_bits[b, :, i, : pb + i + 1].all()
                assert not got_bits[b, :, i, pb + i + 1:].any()
            K, V = inp.seq_k(b), inp.seq_v(b)
            picks = sorted({nqb - 1} | set(rng.choice(nqb, size=min(nqb, DENSE_BLOCKS),
                                                      replace=False).tolist()))
            a = int(inp.cu_seqlens_q[b])
            for i in picks:
                r0, r1 = max(0, i * B - off), min(Lq, (i + 1) * B - off)
                Qb = inp._deq(inp.q[a + r0: a + r1], inp.q_scale)
                parts = list(ex.map(lambda h: O.dense_query_block(Qb, K, V, P + r0, [h]),
                                    range(shape.Hq)))
                ref = np.stack([x.reshape(r1 - r0, -1) for x in parts], axis=1)
                got = pr.out[a + r0: a + r1].double().cpu().numpy()
                H.assert_close(got, ref, fp8, f"w{cid} dense seq {b} block {i}")
                rows += (r1 - r0) * shape.Hq
    assert rows >= DENSE_BLOCKS * B * shape.Hq
    print(f"w{cid}-{dtype} dense: rows compared={rows}")
