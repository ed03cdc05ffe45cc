"""e4m3 KV caches quantised per key block (one K and one V scale per
sequence, key block and KV head, given as factors of the per-head scale):
block means, scores, masks and the corrected attention against the fp64
oracle on the dequantised inputs, paged and contiguous, with a resident
prefix, a decode row and a partial last block; the block-mean cache
bit-identical to recomputing; the host-side argument rules.  The kernel folds
each block's V factor into P before its e4m3 rounding (FlashPrefill V2
popular explainer, section 2.3: E4M3 input/output)."""
import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

CASES = {
    "paged64": dict(lens_q=[700, 300], page_size=64),
    "contiguous": dict(lens_q=[900]),
    "prefix_decode_paged": dict(lens_q=[333, 1, 128], lens_k=[333 + 512, 1 + 700, 128 + 77],
                                page_size=64),
    "g8_paged128": dict(lens_q=[520, 260], Hq=16, Hkv=2, page_size=128),
}


def _inputs(name):
    kw = dict(CASES[name])
    kw.setdefault("Hq", 8)
    kw.setdefault("Hkv", 2)
    return synth.make_inputs(H.small_shape(dtype="fp8", kv_scales="block", seed=61, drop=0.6,
                                           **kw))


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_block_scaled_prefill_matches_oracle(name):
    inp = _inputs(name)
    s = inp.shape
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, s.drop)
    pr = H.problem(inp, out_fill=float("nan"), ws_fill=0xFF)
    pr.prefill(tau)
    pr.check()
    L = pr.layout()
    kbar = pr.ws_view("kbar", torch.float32, (inp.num_seqs, s.Hkv, L.nkb_max, s.d)).cpu().double().numpy()
    vbar = pr.ws_view("vbar", torch.float32, (inp.num_seqs, s.Hkv, L.nkb_max, s.d)).cpu().double().numpy()
    got_bits = H.gpu_bits(pr, inp)
    for b in range(inp.num_seqs):
        kb, vb, cnt, S, pb = orc[b]
        nkb = kb.shape[1]
        np.testing.assert_allclose(kbar[b, :, :nkb], kb, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(vbar[b, :, :nkb], vb, rtol=1e-5, atol=1e-5)
        keep = O.mask(S, pb, tau)
        assert (got_bits[b, :, : S.shape[1], :nkb] == keep.astype(bool)).all(), f"seq {b} mask"
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        got = H.out_seq(pr, inp, b).reshape(ref.shape)
        assert np.isfinite(got).all()
        H.assert_close(got, ref, True, f"{name} seq {b}")


@pytest.mark.gpu
def test_block_scaled_mean_cache_is_bit_identical():
    """Chunked prefill with the block-mean cache: the cache holds the raw means
    of the stored values and the factors are applied when they are read, so
    the workspace equals the uncached one bit for bit."""
    inp = _inputs("prefix_decode_paged")
    s = inp.shape
    pr = H.problem(inp)
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    pr.check()
    L = pr.layout()
    n = L.vbar_op + inp.num_seqs * s.Hkv * L.nkb_max * s.d * 2 - L.kbar
    ref = pr.workspace[L.kbar: L.kbar + n].clone()
    nblk = [-(-Lk // s.B) for Lk in s.lens_k]
    table = torch.full((len(nblk), max(nblk)), -1, dtype=torch.int32)
    off = 0
    for b, m in enumerate(nblk):
        table[b, :m] = torch.arange(off, off + m, dtype=torch.int32)
        off += m
    table = table.cuda()
    cache = torch.zeros((off, 2, s.Hkv, s.d), dtype=torch.float32, device="cuda")
    # fill every slot as the earlier chunks would have: the same K/V with the
    # whole sequences as the call's rows (no prefix), then the call itself
    cu_full = torch.tensor(np.concatenate([[0], np.cumsum(s.lens_k)]), dtype=torch.int32,
                           device="cuda")
    fill = fp2.make_problem(pr.q, pr.k, pr.v, cu_full, Hq=s.Hq, Hkv=s.Hkv, d=s.d, block=s.B,
                            dtype=pr.dtype, max_seqlen_q=max(s.lens_k),
                            max_seqlen_k=max(s.lens_k), seqlens_k=inp.seqlens_k.cuda(),
                            page_table=pr.page_table, page_size=s.page_size,
                            q_scale=inp.q_scale.cuda(), k_scale=inp.k_scale.cuda(),
                            v_scale=inp.v_scale.cuda(),
                            k_block_factor=inp.k_block_factor.contiguous().cuda(),
                            v_block_factor=inp.v_block_factor.contiguous().cuda())
    fill.params.total_q = int(sum(s.lens_k))
    fp2.blockmean_cached(pr.k, pr.v, pr.page_table, cu_full, table, max(nblk), cache, off, s.B,
                         pr.dtype, fill.params)
    fill.check()
    for _ in range(2):
        fp2.blockmean_cached(pr.k, pr.v, pr.page_table, pr.cu_seqlens, table, max(nblk), cache,
                             off, s.B, pr.dtype, pr.params)
        pr.check()
        assert torch.equal(pr.workspace[L.kbar: L.kbar + n], ref)


def test_block_factors_need_e4m3_and_the_two_tile_kernel():
    """Host-side rules (no GPU needed): factors with bf16 inputs, only one of
    the two arrays, or the one-tile kernel are rejected before any launch."""
    P = fp2.Params()
    P.num_seqs, P.num_q_heads, P.num_kv_heads, P.head_dim = 1, 8, 2, 128
    P.total_q = P.total_k = P.max_seqlen_q = P.max_seqlen_k = 256
    fake = 1 << 20
    P.workspace, P.workspace_bytes = 256, 1 << 40
    P.q_scale = P.k_scale = P.v_scale = fake
    lib = fp2.lib()
    import ctypes

    def call(dtype):
        return lib.fp2_attn(fake, fake, fake, None, fake, None, 128, dtype, fake,
                            ctypes.byref(P))
    P.k_block_factor = P.v_block_factor = fake
    assert call(fp2.FP2_BF16) == fp2.FP2_ERR_INVALID_ARG
    P.v_block_factor = None
    assert call(fp2.FP2_FP8_E4M3) == fp2.FP2_ERR_INVALID_ARG
    P.v_block_factor = fake
    P.attn_kernel = 1
    assert call(fp2.FP2_FP8_E4M3) == fp2.FP2_ERR_UNSUPPORTED


def test_generator_block_quantisation():
    """The generator's per-block e4m3 quantisation (CPU): factors in (0, 1]
    with the largest of each head equal to 1, and every block's dequantised
    values within e4m3's rounding of their own block scale."""
    inp = _inputs("paged64")
    s = inp.shape
    for fac in (inp.k_block_factor, inp.v_block_factor):
        f = fac.numpy()
        assert (f > 0).all() and (f <= 1).all()
        np.testing.assert_allclose(f.max(axis=(0, 1)), 1.0)
    for b in range(inp.num_seqs):
        V = inp.seq_v(b)
        nkb = -(-V.shape[0] // s.B)
        for j in range(nkb):
            blk = V[j * s.B:(j + 1) * s.B]
            scale = float(inp.v_scale.double()[0]) * float(inp.v_block_factor[b, j, 0])
            assert np.abs(blk[:, 0]).max() <= 448 * scale * (1 + 1e-6)
            # e4m3 codes: value / scale on the e4m3 grid
            codes = blk[:, 0] / scale
            r = torch.tensor(codes, dtype=torch.float32).to(torch.float8_e4m3fn).double().numpy()
            np.testing.assert_allclose(r, codes, rtol=1e-6, atol=1e-9)


def test_dtype_free_entry_points_accept_fp8_formats():
    """fp2_mask and fp2_calibrate_tau take no dtype, so per-block factors and
    e4m3 output without out_scale (valid for e4m3 inputs) must not be judged
    as if the inputs were bf16.  Without a GPU the launch itself fails with
    FP2_ERR_CUDA; what matters is that it is not an argument error."""
    import ctypes
    P = fp2.Params()
    P.num_seqs, P.num_q_heads, P.num_kv_heads, P.head_dim = 1, 8, 2, 128
    P.total_q = P.total_k = P.max_seqlen_q = P.max_seqlen_k = 256
    P.workspace, P.workspace_bytes = 256, 1 << 40
    fake = 1 << 20
    P.q_scale = P.k_scale = P.v_scale = fake
    P.k_block_factor = P.v_block_factor = fake
    P.out_dtype = fp2.FP2_FP8_E4M3
    st = fp2.lib().fp2_mask(fake, ctypes.c_float(1.0), 128, ctypes.byref(P))
    assert st != fp2.FP2_ERR_INVALID_ARG


@pytest.mark.gpu
def test_calibrate_tau_with_block_factors():
    inp = _inputs("paged64")
    s = inp.shape
    pr = H.problem(inp)
    fp2.blockmean(pr.k, pr.v, pr.page_table, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    fp2.score(pr.q, pr.cu_seqlens, s.B, pr.dtype, pr.params)
    tau = fp2.calibrate_tau(pr.cu_seqlens, s.B, 0.6, pr.params)
    fp2.mask(pr.cu_seqlens, tau, s.B, pr.params)
    pr.check()
    assert np.isfinite(tau)
