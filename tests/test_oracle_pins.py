"""Pins of the fp64 oracle to things other than itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them; the
mutation tests at the bottom compile such slips into the oracle and check
exactly that.

* dense routine == torch's scaled_dot_product_attention (a library routine);
* tau = +inf (every block kept) == brute-force dense causal attention;
* correction exact when every non-forced block has constant K and V rows
  (then a dropped block IS n_j copies of one token -- the reason the
  pseudo-token form is the one taken for the pages' mean correction);
* uniform attention (q = 0): output = mean of V over the causal prefix for
  every tau (closed form);
* a hand-worked 3-block case with one dropped block;
* block means / pooled queries / scores == numpy mean and einsum, with the
  query blocks cut at absolute positions when the prefix is not a multiple
  of the block (decode rows, arbitrary chunk boundaries);
* a decode row given the full prefill's mask equals the full prefill's last
  row;
* threshold: hand-made score rows with obvious kept sets (max-based dynamic
  thresholding of the FlashPrefill V2 abstract, plus the forced first and
  diagonal blocks);
* weights of kept tokens and dropped-block pseudo-tokens sum to one.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


def rand_seq(rng, Lq, Lk, Hq, Hkv, d, scale=1.0):
    Q = rng.standard_normal((Lq, Hq, d)) * scale
    K = rng.standard_normal((Lk, Hkv, d)) * scale
    V = rng.standard_normal((Lk, Hkv, d))
    return Q, K, V


def sdpa_dense(Q, K, V):
    """torch SDPA (fp64, CPU) with an explicit bottom-right causal mask."""
    Lq, Hq, d = Q.shape
    Lk, Hkv, _ = K.shape
    G = Hq // Hkv
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    P = Lk - Lq
    allowed = (torch.arange(Lk)[None, :] <= (P + torch.arange(Lq))[:, None])
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed)
    return o[0].permute(1, 0, 2).numpy()  # [Lq, Hq, d]


SHAPES = [  # Lq, Lk, Hq, Hkv, d, B
    (37, 37, 2, 1, 8, 8),
    (64, 64, 4, 2, 16, 16),
    (29, 61, 4, 1, 8, 8),     # prefix of 32 (4 blocks of 8), ragged tail
    (50, 50, 8, 8, 4, 4),
    (9, 9, 1, 1, 3, 16),      # one partial block
    (1, 61, 4, 1, 8, 8),      # a decode row: one query at position 60 (block 7, offset 4)
    (13, 50, 2, 1, 8, 8),     # prefix 37: the first query block holds 3 rows
    (5, 23, 4, 2, 4, 16),     # prefix 18: the whole call inside one block
    (40, 47, 4, 2, 8, 8),     # prefix 7: first query block of 1 row, ragged tail
]


@pytest.mark.parametrize("shape", SHAPES)
def test_dense_routine_matches_torch_sdpa(shape):
    Lq, Lk, Hq, Hkv, d, B = shape
    rng = np.random.default_rng(1)
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d)
    rows, heads = O.all_rows(Lq, Hq)
    got = O.dense_rows(Q, K, V, rows, heads).reshape(Lq, Hq, d)
    np.testing.assert_allclose(got, sdpa_dense(Q, K, V), rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", SHAPES)
def test_dense_query_block_matches_the_brute_force(shape):
    """The matrix-product form of dense causal attention (used to check long
    dense runs block by block) against the per-row brute force, on every
    block of each shape, partial first and last blocks included."""
    Lq, Lk, Hq, Hkv, d, B = shape
    rng = np.random.default_rng(3)
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d)
    P = Lk - Lq
    rows, heads = O.all_rows(Lq, Hq)
    ref = O.dense_rows(Q, K, V, rows, heads).reshape(Lq, Hq, d)
    t = 0
    while t < Lq:
        t1 = min(Lq, ((P + t) // B + 1) * B - P)  # the end of the absolute block holding t
        got = O.dense_query_block(Q[t:t1], K, V, P + t).reshape(t1 - t, Hq, d)
        np.testing.assert_allclose(got, ref[t:t1], rtol=0, atol=1e-12)
        sub = np.array([Hq - 1, 0], dtype=np.int32)
        got_sub = O.dense_query_block(Q[t:t1], K, V, P + t, sub).reshape(t1 - t, 2, d)
        np.testing.assert_allclose(got_sub, ref[t:t1][:, sub], rtol=0, atol=1e-12)
        t = t1


@pytest.mark.parametrize("shape", SHAPES)
def test_keep_all_equals_dense(shape):
    Lq, Lk, Hq, Hkv, d, B = shape
    rng = np.random.default_rng(2)
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d, scale=1.5)
    r = O.prefill_seq(Q, K, V, B, math.inf)
    causal = ~np.isnan(r.S)
    assert r.keep[causal].all() and not r.keep[~causal].any()
    dense = O.dense_rows(Q, K, V, r.rows, r.heads)
    np.testing.assert_allclose(r.out, dense, rtol=0, atol=1e-12)


def constant_block_seq(rng, Lq, Lk, Hq, Hkv, d, B):
    """K and V rows constant inside every key block (block values random)."""
    nkb = -(-Lk // B)
    kb = rng.standard_normal((nkb, Hkv, d)) * 1.3
    vb = rng.standard_normal((nkb, Hkv, d))
    idx = np.arange(Lk) // B
    K = kb[idx].copy()
    V = vb[idx].copy()
    Q = rng.standard_normal((Lq, Hq, d)) * 1.3
    return Q, K, V


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("tau", [-1e9, 0.0, 0.3, 1.0, 3.0])
def test_correction_exact_for_constant_blocks(shape, tau):
    Lq, Lk, Hq, Hkv, d, B = shape
    rng = np.random.default_rng(3)
    Q, K, V = constant_block_seq(rng, Lq, Lk, Hq, Hkv, d, B)
    r = O.prefill_seq(Q, K, V, B, tau)
    dense = O.dense_rows(Q, K, V, r.rows, r.heads)
    np.testing.assert_allclose(r.out, dense, rtol=0, atol=1e-12)
    if tau == -1e9:
        # only block 0 and the diagonal survive
        nqb = r.keep.shape[1]
        P = Lk - Lq
        for i in range(nqb):
            iabs = P // B + i
            kept = set(np.nonzero(r.keep[0, i])[0].tolist())
            assert kept == {0, iabs}


def test_correction_not_exact_for_general_blocks():
    """Sanity: the constant-block pin is not vacuous -- with ordinary rows and
    blocks dropped, the corrected output differs from dense."""
    rng = np.random.default_rng(4)
    Q, K, V = rand_seq(rng, 64, 64, 2, 1, 8, scale=1.5)
    r = O.prefill_seq(Q, K, V, 8, -1e9)
    dense = O.dense_rows(Q, K, V, r.rows, r.heads)
    assert np.abs(r.out - dense).max() > 1e-3


@pytest.mark.parametrize("tau", [-1e9, 0.5, math.inf])
def test_uniform_attention_closed_form(tau):
    """q = 0: every logit is 0, a dropped block weighs n_j, so the output is
    the plain mean of V over positions 0..p whatever is kept."""
    rng = np.random.default_rng(5)
    Lq, Lk, Hq, Hkv, d, B = 21, 45, 2, 1, 6, 8
    _, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d)
    Q = np.zeros((Lq, Hq, d))
    # pooled query is 0 -> every score 0 -> ties keep everything unless tau < 0
    r = O.prefill_seq(Q, K, V, B, tau)
    P = Lk - Lq
    out = r.out.reshape(Lq, Hq, d)
    for t in range(Lq):
        want = V[: P + t + 1, 0, :].mean(axis=0)
        for h in range(Hq):
            np.testing.assert_allclose(out[t, h], want, rtol=0, atol=1e-13)


def test_three_block_worked_example():
    """B = 2, d = 1, one head, 6 tokens.  Keys: block0 = [1, 1],
    block1 = [ln 4, -ln 4] (mean 0), block2 = [1, 1]; queries all 1; values
    v = [1, 2, 4, 6, 3, 5].  Query block 2 (rows 4, 5) pools to 1, so its
    scores are s20 = 1, s21 = 0, s22 = 1; with tau = 0.5 block 1 is dropped
    (0 < 1 - 0.5) and enters as one pseudo-token of logit 0 + ln 2 with value
    mean(4, 6) = 5.  Row 4 then weighs tokens 0, 1, 4 by e each and the
    pseudo-token by 2: out = (e*1 + e*2 + e*3 + 2*5) / (3e + 2).  Row 5 adds
    token 5 (logit 1, value 5): (e*(1+2+3+5) + 10) / (4e + 2).  Query block 1
    keeps blocks 0 and 1 (both forced), so rows 2, 3 are dense."""
    e = math.e
    ln4 = math.log(4.0)
    K = np.array([1, 1, ln4, -ln4, 1, 1], dtype=np.float64).reshape(6, 1, 1)
    V = np.array([1, 2, 4, 6, 3, 5], dtype=np.float64).reshape(6, 1, 1)
    Q = np.ones((6, 1, 1))
    r = O.prefill_seq(Q, K, V, 2, 0.5)
    assert r.keep[0, 2].tolist() == [1, 0, 1]
    np.testing.assert_allclose(r.S[0, 2], [1.0, 0.0, 1.0], atol=1e-15)
    out = r.out.reshape(6)
    assert out[4] == pytest.approx((6 * e + 10) / (3 * e + 2), abs=1e-14)
    assert out[5] == pytest.approx((11 * e + 10) / (4 * e + 2), abs=1e-14)
    # row 3 (block 1, dense over tokens 0..3): logits 1, 1, ln4, -ln4
    w = np.array([e, e, 4.0, 0.25])
    assert out[3] == pytest.approx((w * [1, 2, 4, 6]).sum() / w.sum(), abs=1e-14)
    assert out[0] == pytest.approx(1.0, abs=1e-15)


def test_blockmean_pool_score_match_numpy():
    rng = np.random.default_rng(6)
    Lq, Lk, Hq, Hkv, d, B = 45, 77, 4, 2, 8, 16
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d)
    kbar, vbar, cnt = O.blockmean(K, V, B)
    nkb = -(-Lk // B)
    assert cnt.tolist() == [16, 16, 16, 16, 13]
    for j in range(nkb):
        np.testing.assert_allclose(kbar[:, j], K[j * B:(j + 1) * B].mean(axis=0), atol=1e-14)
        np.testing.assert_allclose(vbar[:, j], V[j * B:(j + 1) * B].mean(axis=0), atol=1e-14)
    qbar = O.pool_q(Q, B)
    for i in range(-(-Lq // B)):
        np.testing.assert_allclose(qbar[:, i], Q[i * B:(i + 1) * B].mean(axis=0), atol=1e-14)
    P = Lk - Lq  # 32 -> 2 prefix blocks
    S = O.score(qbar, kbar, P // B)
    G = Hq // Hkv
    full = np.einsum("hid,hjd->hij", qbar, np.repeat(kbar, G, axis=0)) / math.sqrt(d)
    for i in range(S.shape[1]):
        iabs = P // B + i
        np.testing.assert_allclose(S[:, i, : iabs + 1], full[:, i, : iabs + 1], atol=1e-13)
        assert np.isnan(S[:, i, iabs + 1:]).all()


@pytest.mark.parametrize("Lq,P,B", [(1, 60, 8), (13, 37, 8), (5, 18, 16), (40, 7, 8),
                                     (24, 16, 8)])
def test_pool_q_cuts_blocks_at_absolute_positions(Lq, P, B):
    """The call's query blocks follow the absolute blocks: row t belongs to
    block (P + t) // B - P // B, and each pooled query is the numpy mean of
    exactly those rows."""
    rng = np.random.default_rng(13)
    Q = rng.standard_normal((Lq, 3, 5))
    qbar = O.pool_q(Q, B, P % B)
    lab = (P + np.arange(Lq)) // B - P // B
    assert qbar.shape[1] == lab[-1] + 1
    for i in range(qbar.shape[1]):
        np.testing.assert_allclose(qbar[:, i], Q[lab == i].mean(axis=0), rtol=0, atol=1e-14)


def test_decode_row_keeps_and_corrects_like_a_prefill_row():
    """A decode row (Lq = 1) at position p is the last row of the same
    sequence's full prefill when the masks agree: with the mask of the full
    prefill's last query block given explicitly, the two outputs coincide
    (same kept tokens, same pseudo-tokens)."""
    rng = np.random.default_rng(14)
    L, Hq, Hkv, d, B = 77, 4, 2, 8, 8
    Q, K, V = rand_seq(rng, L, L, Hq, Hkv, d, scale=1.5)
    full = O.prefill_seq(Q, K, V, B, 0.4)
    assert full.keep.sum() < np.isfinite(full.S).sum()  # something is dropped
    keep_last = full.keep[:, -1:, :]
    one = O.prefill_seq(Q[-1:], K, V, B, 0.4, keep=keep_last)
    want = full.out.reshape(L, Hq, d)[-1]
    np.testing.assert_allclose(one.out.reshape(Hq, d), want, rtol=0, atol=1e-13)
    # and the decode row's own mask is scored with its own query, not the block mean
    own = O.prefill_seq(Q[-1:], K, V, B, 0.4)
    G = Hq // Hkv
    qs = np.einsum("hd,hjd->hj", Q[-1], np.repeat(own.kbar, G, axis=0)) / math.sqrt(d)
    np.testing.assert_allclose(own.S[:, 0, :], qs, rtol=0, atol=1e-13)


def test_mask_hand_made_rows():
    # one head, one query block at absolute index 4 (prefix of 4 blocks)
    S = np.array([[[5.0, 1.0, 4.5, 0.0, 2.0, np.nan]]])
    assert O.mask(S, 4, 1.0)[0, 0].tolist() == [1, 0, 1, 0, 1, 0]
    # inclusive threshold: s == m - tau is kept
    assert O.mask(S, 4, 3.0)[0, 0].tolist() == [1, 0, 1, 0, 1, 0]
    assert O.mask(S, 4, 3.0000001)[0, 0].tolist() == [1, 0, 1, 0, 1, 0]
    assert O.mask(S, 4, 4.0)[0, 0].tolist() == [1, 1, 1, 0, 1, 0]
    assert O.mask(S, 4, math.inf)[0, 0].tolist() == [1, 1, 1, 1, 1, 0]
    assert O.mask(S, 4, -100.0)[0, 0].tolist() == [1, 0, 0, 0, 1, 0]
    # the row maximum counts the forced blocks too; the max itself is kept
    S2 = np.array([[[0.0, 3.0, 2.5, 9.0, np.nan, np.nan]]])
    assert O.mask(S2, 3, 0.5)[0, 0].tolist() == [1, 0, 0, 1, 0, 0]
    assert O.mask(S2, 3, 6.2)[0, 0].tolist() == [1, 1, 0, 1, 0, 0]
    assert O.mask(S2, 3, 6.6)[0, 0].tolist() == [1, 1, 1, 1, 0, 0]
    # block 0 is its own diagonal
    S3 = np.array([[[-7.0, np.nan]]])
    assert O.mask(S3, 0, -1.0)[0, 0].tolist() == [1, 0]


def test_weights_sum_to_one():
    rng = np.random.default_rng(7)
    Lq, Lk, Hq, Hkv, d, B = 40, 72, 4, 2, 8, 8
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d, scale=2.0)
    r = O.prefill_seq(Q, K, V, B, 0.7)
    assert (r.keep.sum() < np.isfinite(r.S).sum())  # something was dropped
    _, wsum = O.attn_rows(Q, K, V, r.kbar, r.vbar, r.cnt, r.keep, B, r.rows, r.heads,
                          want_wsum=True)
    np.testing.assert_allclose(wsum, 1.0, rtol=0, atol=1e-12)


def test_tau_for_drop_hits_target_and_guard():
    rng = np.random.default_rng(8)
    Lq, Lk, Hq, Hkv, d, B = 256, 256, 4, 1, 8, 8
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d, scale=1.5)
    kbar, vbar, cnt = O.blockmean(K, V, B)
    S = O.score(O.pool_q(Q, B), kbar, 0)
    total = sum(Hq * (i + 1) for i in range(Lq // B))
    for target in (0.3, 0.5, 0.7):
        tau = O.tau_for_drop([S], [0], target)
        keep = O.mask(S, 0, tau)
        dropped = total - int(keep.sum())
        assert abs(dropped - round(target * total)) <= 1
        tau_g = O.tau_for_drop([S], [0], target, guard=1e-3)
        mg, _ = O.margins([S], [0])
        assert np.abs(mg - tau_g).min() > 1e-3
        dropped_g = total - int(O.mask(S, 0, tau_g).sum())
        assert abs(dropped_g - target * total) < 0.05 * total


# --------------------------------------------------------------------------
# mutation tests: each compiled slip must be caught by at least one pin
# --------------------------------------------------------------------------

def _pins_pass(mutant: int) -> bool:
    rng = np.random.default_rng(9)
    ok = True
    # keep-all vs dense + constant blocks + worked example + mask cases
    Lq, Lk, Hq, Hkv, d, B = 29, 61, 4, 1, 8, 8
    Q, K, V = constant_block_seq(rng, Lq, Lk, Hq, Hkv, d, B)
    r = O.prefill_seq(Q, K, V, B, 0.3, mutant=mutant)
    dense = O.dense_rows(Q, K, V, r.rows, r.heads)
    ok &= np.abs(r.out - dense).max() < 1e-12
    e = math.e
    ln4 = math.log(4.0)
    K3 = np.array([1, 1, ln4, -ln4, 1, 1], dtype=np.float64).reshape(6, 1, 1)
    V3 = np.array([1, 2, 4, 6, 3, 5], dtype=np.float64).reshape(6, 1, 1)
    r3 = O.prefill_seq(np.ones((6, 1, 1)), K3, V3, 2, 0.5, mutant=mutant)
    ok &= abs(r3.out.reshape(6)[4] - (6 * e + 10) / (3 * e + 2)) < 1e-14
    S = np.array([[[5.0, 1.0, 4.5, 0.0, 2.0, np.nan]]])
    ok &= O.mask(S, 4, 3.0, mutant=mutant)[0, 0].tolist() == [1, 0, 1, 0, 1, 0]
    Qr, Kr, Vr = rand_seq(rng, 45, 77, 4, 2, 8)
    kbar, _, _ = O.blockmean(Kr, Vr, 16, mutant=mutant)
    ok &= np.abs(kbar[:, 1] - Kr[16:32].mean(axis=0)).max() < 1e-14
    # a prefix that is not a multiple of the block: constant blocks, only the
    # forced blocks kept, still exact; pooled queries follow absolute blocks
    Qu, Ku, Vu = constant_block_seq(rng, 29, 63, 4, 1, 8, 8)
    ru = O.prefill_seq(Qu, Ku, Vu, 8, -1e9, mutant=mutant)
    ok &= np.abs(ru.out - O.dense_rows(Qu, Ku, Vu, ru.rows, ru.heads)).max() < 1e-12
    qb = O.pool_q(Qu, 8, 34 % 8, mutant=mutant)
    ok &= qb.shape[1] == 4 and np.abs(qb[:, 0] - Qu[:6].mean(axis=0)).max() < 1e-14
    return bool(ok)


def test_pins_pass_on_the_oracle():
    assert _pins_pass(0)


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6])
def test_pins_catch_mutant(mutant):
    assert not _pins_pass(mutant)


# --------------------------------------------------------------------------
# group-shared masks (a variant: one mask per KV group, scored with the
# group-mean pooled query)
# --------------------------------------------------------------------------

def test_group_masks_equal_head_masks_when_heads_agree():
    """If the G query heads of a group carry identical queries, the group
    mean is each head's pooled query: group masks = per-head masks, and the
    outputs agree."""
    rng = np.random.default_rng(12)
    Lq, Lk, Hq, Hkv, d, B = 70, 102, 4, 2, 8, 8
    Q, K, V = rand_seq(rng, Lq, Lk, Hq, Hkv, d, scale=1.5)
    Q[:, 1] = Q[:, 0]
    Q[:, 3] = Q[:, 2]
    a = O.prefill_seq(Q, K, V, B, 0.6)
    g = O.prefill_seq(Q, K, V, B, 0.6, group_masks=True)
    assert (a.keep == g.keep).all()
    np.testing.assert_allclose(a.out, g.out, atol=1e-13)


def test_group_masks_use_the_mean_query():
    """Hand-made: one KV head, two query heads, d = 1, B = 2, 6 tokens.
    Queries: head 0 = +2, head 1 = -1 (group mean +0.5).  Keys: block0 = [1, 1],
    block1 = [-3, -3], block2 = [0.2, 0.2].  Query block 2 scores: per head 0:
    (2, -6, 0.4), per head 1: (-1, 3, -0.2), group: (0.5, -1.5, 0.1).  With
    tau = 1 the per-head masks are head 0: {0, 2}, head 1: {1 (the max), 0 and
    2 forced} -> [1,1,1]; the group mask keeps {0, 2} (-1.5 < 0.5 - 1) for both
    heads."""
    K = np.array([1, 1, -3, -3, 0.2, 0.2], dtype=np.float64).reshape(6, 1, 1)
    V = np.arange(6, dtype=np.float64).reshape(6, 1, 1)
    Q = np.zeros((6, 2, 1))
    Q[:, 0] = 2.0
    Q[:, 1] = -1.0
    a = O.prefill_seq(Q, K, V, 2, 1.0)
    g = O.prefill_seq(Q, K, V, 2, 1.0, group_masks=True)
    assert a.keep[0, 2].tolist() == [1, 0, 1] and a.keep[1, 2].tolist() == [1, 1, 1]
    assert g.keep[0, 2].tolist() == [1, 0, 1] and g.keep[1, 2].tolist() == [1, 0, 1]
    np.testing.assert_allclose(g.S[:, 2], [[0.5, -1.5, 0.1]] * 2, atol=1e-15)
