"""GPU parity: every stage of the CUDA path, called through the C ABI,
against the fp64 oracle on the same seeded inputs.

Bars: block means and scores within fp32 rounding of the oracle; masks bit
exact (tau is placed in a gap of the oracle's margins at least 2e-3 wide, so
no score lies within 1e-3 of the threshold); outputs within rel-L2 5e-3 and
max-abs 2e-2 (bf16) or rel-L2 5e-2 (e4m3, against the oracle on the
dequantised inputs)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu

CASES = {
    # name: (shape kwargs)
    "tiny_1k_d64_b64": dict(lens_q=[1024], Hq=4, Hkv=1, d=64, B=64, latents="per_block"),
    "ragged_2k_g4": dict(lens_q=[2125], Hq=8, Hkv=2),
    "ragged_2k_g4_fp8": dict(lens_q=[2125], Hq=8, Hkv=2, dtype="fp8"),
    "g1_b128": dict(lens_q=[777], Hq=4, Hkv=4),
    "g2_b64_d128": dict(lens_q=[1000], Hq=4, Hkv=2, B=64),
    "g8_d64": dict(lens_q=[900], Hq=16, Hkv=2, d=64),
    "varlen_paged64": dict(lens_q=[300, 1000, 129, 1, 2000], Hq=8, Hkv=2, page_size=64),
    "varlen_paged64_fp8": dict(lens_q=[300, 1000, 129, 1, 2000], Hq=8, Hkv=2, page_size=64,
                               dtype="fp8"),
    "varlen_paged16_b64": dict(lens_q=[250, 700], Hq=8, Hkv=4, B=64, page_size=16),
    "varlen_paged256": dict(lens_q=[650, 1300], Hq=8, Hkv=2, page_size=256),
    "chunk_prefix_g8": dict(lens_q=[700], lens_k=[1024 + 700], Hq=16, Hkv=2, page_size=64),
    "chunk_prefix_g8_fp8": dict(lens_q=[700], lens_k=[1024 + 700], Hq=16, Hkv=2, page_size=64,
                                dtype="fp8"),
    "chunk_prefix_short": dict(lens_q=[60, 128], lens_k=[512 + 60, 256 + 128], Hq=8, Hkv=2,
                               page_size=32),
    # decode rows (Lq = 1) and chunks whose prefix is not a multiple of the
    # block, mixed with ordinary prefill rows in one batch; prefixes 3000,
    # 963, 1013, 127, 128, 0 (offsets 56, 67, 117, 127, 0, 0 into the block)
    "mixed_decode_paged64": dict(lens_q=[1, 37, 700, 1, 1, 300],
                                 lens_k=[3001, 1000, 1713, 128, 129, 300], Hq=8, Hkv=2,
                                 page_size=64),
    "mixed_decode_paged64_fp8": dict(lens_q=[1, 37, 700, 1, 1, 300],
                                     lens_k=[3001, 1000, 1713, 128, 129, 300], Hq=8, Hkv=2,
                                     page_size=64, dtype="fp8"),
    "mixed_decode_g8": dict(lens_q=[1, 45, 250], lens_k=[777, 1000, 2503], Hq=16, Hkv=2),
    "mixed_decode_g1": dict(lens_q=[1, 200, 5], lens_k=[2000, 1290, 133], Hq=4, Hkv=4),
    "mixed_decode_b64_d64": dict(lens_q=[1, 90, 3], lens_k=[1500, 700, 67], Hq=4, Hkv=2, d=64,
                                 B=64, page_size=16),
}


def make_inputs(name):
    kw = dict(CASES[name])
    return synth.make_inputs(H.small_shape(**kw))


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    inp = make_inputs(request.param)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, inp.shape.drop)
    return request.param, inp, orc, tau


def test_blockmean_and_scores(case):
    name, inp, orc, tau = case
    pr = H.problem(inp, ws_fill=0xFF)
    s = inp.shape
    dt = pr.dtype
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, dt, pr.params)
    fp2.score(pr.q, pr.cu_seqlens, s.B, dt, pr.params)
    pr.check()
    L = pr.layout()
    S_ = inp.num_seqs
    kbar = pr.ws_view("kbar", torch.float32, (S_, s.Hkv, L.nkb_max, s.d)).cpu().double().numpy()
    vbar = pr.ws_view("vbar", torch.float32, (S_, s.Hkv, L.nkb_max, s.d)).cpu().double().numpy()
    sc = pr.ws_view("scores", torch.float32, (S_, s.Hq, L.nqb_max, L.nkb_max)).cpu().double().numpy()
    for b, (kb, vb, cnt, S, pb) in enumerate(orc):
        nkb = kb.shape[1]
        np.testing.assert_allclose(kbar[b, :, :nkb], kb, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(vbar[b, :, :nkb], vb, rtol=1e-5, atol=1e-5)
        assert (kbar[b, :, nkb:] == 0).all() and (vbar[b, :, nkb:] == 0).all()
        for i in range(S.shape[1]):
            iabs = pb + i
            np.testing.assert_allclose(sc[b, :, i, : iabs + 1], S[:, i, : iabs + 1],
                                       rtol=1e-5, atol=2e-4)


def test_mask_bit_exact(case):
    name, inp, orc, tau = case
    pr = H.problem(inp, ws_fill=0xFF)
    s = inp.shape
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    fp2.score(pr.q, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    fp2.mask(pr.cu_seqlens, tau, s.B, pr.params)
    pr.check()
    got = H.gpu_bits(pr, inp)
    L = pr.layout()
    idx = pr.ws_view("kept_idx", torch.int32, (inp.num_seqs, s.Hq, L.nqb_max, L.nkb_max)).cpu().numpy()
    cnt = pr.ws_view("kept_cnt", torch.int32, (inp.num_seqs, s.Hq, L.nqb_max)).cpu().numpy()
    keeps = []
    for b, (kb, vb, c, S, pb) in enumerate(orc):
        keep = O.mask(S, pb, tau)
        keeps.append(keep)
        nqb, nkb = S.shape[1], S.shape[2]
        assert (got[b, :, :nqb, :nkb] == keep.astype(bool)).all()
        assert not got[b, :, :nqb, nkb:].any()
        for h in range(s.Hq):
            for i in range(nqb):
                want = np.nonzero(keep[h, i])[0]
                assert cnt[b, h, i] == want.size
                assert (idx[b, h, i, : want.size] == want).all()
    frac = H.drop_fraction(keeps, orc)
    assert frac > 0.2 or inp.shape.lens_q == [1] or max(inp.shape.lens_k) <= 6 * s.B


def test_attn_on_oracle_mask(case):
    """fp2_attn alone, fed the oracle's mask: isolates the attention kernel."""
    name, inp, orc, tau = case
    pr = H.problem(inp, out_fill=float("nan"))
    s = inp.shape
    fp8 = s.dtype == "fp8"
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    keeps = [O.mask(r[3], r[4], tau) for r in orc]
    bits = H.bits_from_keep(keeps, inp, pr.layout()).cuda()
    fp2.attn(pr.q, pr.k, pr.v, pr.page_table, pr.cu_seqlens, bits, s.B, pr.dtype, pr.out,
             pr.params)
    pr.check()
    for b in range(inp.num_seqs):
        if s.lens_q[b] == 0:
            continue
        ref, _, _ = H.oracle_out(inp, b, orc[b], keeps[b])
        got = H.out_seq(pr, inp, b).reshape(ref.shape)
        assert np.isfinite(got).all()
        H.assert_close(got, ref, fp8, f"{name} seq {b}")


def test_prefill_end_to_end(case):
    name, inp, orc, tau = case
    pr = H.problem(inp, out_fill=float("nan"), ws_fill=0xFF)
    s = inp.shape
    fp8 = s.dtype == "fp8"
    pr.prefill(tau)
    pr.check()
    for b in range(inp.num_seqs):
        if s.lens_q[b] == 0:
            continue
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        got = H.out_seq(pr, inp, b).reshape(ref.shape)
        H.assert_close(got, ref, fp8, f"{name} seq {b}")


@pytest.mark.parametrize("name", ["tiny_1k_d64_b64", "varlen_paged64", "chunk_prefix_g8",
                                  "ragged_2k_g4_fp8", "mixed_decode_paged64", "mixed_decode_g1"])
def test_keep_all_is_dense_attention(name):
    inp = make_inputs(name)
    pr = H.problem(inp)
    pr.prefill(math.inf)
    pr.check()
    fp8 = inp.shape.dtype == "fp8"
    for b in range(inp.num_seqs):
        Q, K, V = inp.seq_q(b), inp.seq_k(b), inp.seq_v(b)
        rows, heads = O.all_rows(Q.shape[0], Q.shape[1])
        ref = O.dense_rows(Q, K, V, rows, heads).reshape(Q.shape)
        H.assert_close(H.out_seq(pr, inp, b), ref, fp8, f"{name} dense seq {b}")


def test_nan_in_page_tails_and_workspace_does_not_leak():
    """Stale page contents past a sequence's end (here NaN) must not reach
    any output; nor may unwritten workspace (filled with NaN bytes)."""
    inp = make_inputs("varlen_paged64")
    nan = torch.tensor(float("nan")).to(inp.k.dtype)
    ps = inp.k.shape[1]
    for b in range(inp.num_seqs):
        Lk = inp.shape.lens_k[b]
        last = (Lk - 1) // ps
        phys = int(inp.page_table[b, last])
        tail = Lk - last * ps
        inp.k[phys, tail:] = nan
        inp.v[phys, tail:] = nan
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.6)
    pr = H.problem(inp, out_fill=float("nan"), ws_fill=0xFF)
    pr.prefill(tau)
    pr.check()
    for b in range(inp.num_seqs):
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        got = H.out_seq(pr, inp, b).reshape(ref.shape)
        assert np.isfinite(got).all()
        H.assert_close(got, ref, False, f"seq {b}")


def test_empty_sequence_in_batch():
    inp = synth.make_inputs(H.small_shape([300, 0, 129], Hq=8, Hkv=2, page_size=64))
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.5)
    pr = H.problem(inp, out_fill=float("nan"))
    pr.prefill(tau)
    pr.check()
    for b in (0, 2):
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        H.assert_close(H.out_seq(pr, inp, b).reshape(ref.shape), ref, False)


def test_device_errors_are_reported_not_faulted():
    inp = make_inputs("varlen_paged64")
    # a page id out of range
    pr2 = H.problem(inp)
    pt = pr2.page_table.clone()
    pt[2, 0] = 10 ** 6
    pr2.page_table = pt
    pr2.prefill(1.0)
    st, det = fp2.get_status(pr2.params)
    assert st == fp2.FP2_ERR_DEVICE_BOUNDS and det == 3
    assert fp2.get_status(pr2.params) == (fp2.FP2_OK, 0)  # cleared
    # Lk < Lq
    pr3 = H.problem(inp)
    short = inp.seqlens_k.clone()
    short[0] -= 1
    sd = short.cuda()
    pr3.params.seqlens_k = sd.data_ptr()
    pr3.prefill(1.0)
    st, det = fp2.get_status(pr3.params)
    assert st == fp2.FP2_ERR_INVALID_ARG and det == 1


def test_calibrate_tau_matches_target():
    inp = make_inputs("ragged_2k_g4")
    pr = H.problem(inp)
    s = inp.shape
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    fp2.score(pr.q, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    tau = fp2.calibrate_tau(pr.cu_seqlens, s.B, 0.7, pr.params)
    fp2.mask(pr.cu_seqlens, tau, s.B, pr.params)
    pr.check()
    got = H.gpu_bits(pr, inp)
    orc = H.oracle_scores(inp)
    total = sum(s.Hq * (r[4] * r[3].shape[1] + r[3].shape[1] * (r[3].shape[1] + 1) // 2)
                for r in orc)
    kept = int(got.sum())
    assert abs((total - kept) - round(0.7 * total)) <= 2


@pytest.mark.parametrize("name", ["tiny_1k_d64_b64", "varlen_paged64_fp8", "chunk_prefix_g8",
                                  "ragged_2k_g4"])
def test_single_tile_kernel_on_large_groups(name):
    """fp2_params.attn_kernel = 1 routes G*block >= 256 problems to the
    one-tile kernel too, so both attention kernels are checked on the same
    cases."""
    inp = make_inputs(name)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, inp.shape.drop)
    pr = H.problem(inp, out_fill=float("nan"), attn_kernel=1)
    pr.prefill(tau)
    pr.check()
    for b in range(inp.num_seqs):
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        H.assert_close(H.out_seq(pr, inp, b).reshape(ref.shape), ref, inp.shape.dtype == "fp8",
                       f"{name} seq {b}")


@pytest.mark.parametrize("boost,drop", [(6.0, 0.5), (40.0, None)])
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_row_max_jumps_later_in_the_row(boost, drop, dtype):
    """Keys of a later block scaled up so that, after the first kept blocks set
    a row's reference maximum, a later block's logits exceed it by tens (x6)
    or hundreds (x40) of log2 units: the attention kernel's rescale paths
    (scale P down after the fact; redo the item from TMEM) must still match
    the oracle.  The x40 case keeps every block (tau = +inf): a dropped block
    with keys that large would turn the rounding of its mean (the MMA operand
    of the correction) into logit errors of whole units, a different
    question from the rescale paths tested here."""
    shape = H.small_shape([1100], Hq=8, Hkv=2, dtype=dtype, seed=31)
    inp = synth.make_inputs(shape)
    # scale the stored K of block 5 (keeps the stored dtype; the oracle reads
    # the same dequantised values)
    blk = slice(5 * 128, 6 * 128)
    kb = inp._kc[blk].float() * boost
    if dtype == "fp8":
        kb = kb.clamp(-448, 448)
    inp._kc[blk] = kb.to(inp._kc.dtype)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, drop) if drop is not None else float("inf")
    pr = H.problem(inp, out_fill=float("nan"))
    pr.prefill(tau)
    pr.check()
    keep = O.mask(orc[0][3], orc[0][4], tau)
    assert keep[:, 6:, 5].mean() > 0.3  # the boosted block is kept by later rows
    ref, _, _ = H.oracle_out(inp, 0, orc[0], keep)
    got = H.out_seq(pr, inp, 0).reshape(ref.shape)
    assert np.isfinite(got).all()
    H.assert_close(got, ref, dtype == "fp8", f"boost {boost}")
