"""bench.py's useful-work count (the numerator of its TFLOP/s and roofline)
against brute force over the oracle's masks: 4*d flops for every (query row,
kept key token at or before the row) pair, and 4*d for every (query row,
dropped block) pseudo-token, on prefixes aligned and not."""
import math

import numpy as np
import pytest

import bench
from oracle import oracle as O


def brute(keeps, lens_q, lens_k, B, d, Hq):
    kept = corr = 0
    for b, (Lq, Lk) in enumerate(zip(lens_q, lens_k)):
        P = Lk - Lq
        for t in range(Lq):
            p = P + t
            iabs = p // B
            i = iabs - P // B
            for h in range(Hq):
                for j in range(iabs + 1):
                    if keeps[b][h, i, j]:
                        kept += min(p, (j + 1) * B - 1) - j * B + 1
                    else:
                        corr += 1
    return 4.0 * d * kept, 4.0 * d * corr


@pytest.mark.parametrize("lens_q,lens_k,B", [
    ([200], [200], 32),
    ([37, 1, 90], [100, 61, 90], 16),       # prefixes 63 and 60: unaligned, a decode row
    ([64, 50], [64 + 32, 50 + 48], 32),     # aligned prefixes
])
def test_flop_count_matches_brute_force(lens_q, lens_k, B):
    rng = np.random.default_rng(17)
    Hq, Hkv, d = 4, 2, 8
    keeps = []
    nqb_max = max(-(-((Lk - Lq) % B + Lq) // B) for Lq, Lk in zip(lens_q, lens_k))
    cnt = np.zeros((len(lens_q), Hq, nqb_max), dtype=np.int32)
    for b, (Lq, Lk) in enumerate(zip(lens_q, lens_k)):
        Q = rng.standard_normal((Lq, Hq, d)) * 1.5
        K = rng.standard_normal((Lk, Hkv, d)) * 1.5
        V = rng.standard_normal((Lk, Hkv, d))
        r = O.prefill_seq(Q, K, V, B, 0.4)
        keeps.append(r.keep)
        cnt[b, :, : r.keep.shape[1]] = r.keep.sum(axis=2)
    kept, corr, drop = bench.algorithmic_flops(cnt, lens_q, lens_k, B, d)
    want_kept, want_corr = brute(keeps, lens_q, lens_k, B, d, Hq)
    assert kept == pytest.approx(want_kept, rel=0, abs=0.5)
    assert corr == pytest.approx(want_corr, rel=0, abs=0.5)
    assert 0.0 < drop < 1.0 and math.isfinite(drop)


def test_oracle_sample_helpers_cover_every_block_of_a_varlen_batch():
    """bench.py times the oracle block by block (cpu_baseline, the reference
    arm): its per-sequence scores equal the oracle's whole-sequence scores,
    and its per-block attention, stacked over every query block, equals the
    oracle's output for the whole sequence, on a batch with unaligned
    prefixes, a decode row, an empty sequence and more than 64 query blocks
    (the pooling chunk)."""
    from block_sparse_long_blockmean_b200 import synth
    from tests import harness as H
    B = 16
    inp = synth.make_inputs(H.small_shape([1100, 1, 0, 45], [1137, 300, 77, 45], Hq=4, Hkv=2,
                                          d=16, B=B, seed=23))
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.6)
    heads = np.arange(inp.shape.Hq, dtype=np.int32)
    for b in range(inp.num_seqs):
        seq = bench.oracle_seq_scores(inp, b)
        assert seq[6] == orc[b][4]
        np.testing.assert_array_equal(seq[5], orc[b][3])
        if inp.shape.lens_q[b] == 0:
            continue
        keep = O.mask(seq[5], seq[6], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        got = np.concatenate([bench.oracle_block(inp, b, i, seq, keep, heads)
                              for i in range(keep.shape[1])])
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_cpu_baseline_runs_on_a_varlen_batch():
    from block_sparse_long_blockmean_b200 import synth
    from tests import harness as H
    inp = synth.make_inputs(H.small_shape([300, 0, 129], [400, 50, 129], Hq=4, Hkv=2, d=16,
                                          B=16, seed=24))
    tau = H.pick_tau(H.oracle_scores(inp), 0.6)
    cb = bench.cpu_baseline(inp, tau, budget_blocks=3, heads_per_block=2)
    assert cb["value"] > 0 and cb["kind"] == "oracle" and cb["cores"] >= 1
    assert "of all 3 sequence(s)" in cb["sample"]
