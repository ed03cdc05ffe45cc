"""E4M3 output (fp2_params.out_dtype = FP2_FP8_E4M3): out holds O / out_scale[h]
as e4m3.  Dequantised (x out_scale) it must match the oracle within the FP8
tolerance, rel-L2 <= 5e-2 (the e4m3 rounding of the output itself is
~2.7 % rel-RMS).  Default scale with FP8 inputs: the KV head's v_scale, under
which |O| <= 448 so nothing saturates."""
import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kw", [
    dict(lens_q=[2125], Hq=8, Hkv=2, dtype="fp8"),
    dict(lens_q=[700, 300], lens_k=[1024 + 700, 300], Hq=16, Hkv=2, page_size=64, dtype="fp8"),
    dict(lens_q=[1500], Hq=8, Hkv=2, dtype="bf16"),
], ids=["fp8_in_contig", "fp8_in_paged_prefix", "bf16_in"])
def test_e4m3_output(kw):
    inp = synth.make_inputs(H.small_shape(**kw))
    s = inp.shape
    G = s.Hq // s.Hkv
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.7)
    if s.dtype == "fp8":
        scale_h = inp.v_scale.repeat_interleave(G)          # the default the kernel uses
        out_scale = None
    else:
        vmax = torch.stack([inp.v.float()[:, hk].abs().max() for hk in range(s.Hkv)])
        scale_h = (vmax / 448.0).repeat_interleave(G).float()
        out_scale = scale_h.cuda()
    pr = H.problem(inp)
    dev = "cuda"
    pr2 = fp2.make_problem(pr.q, pr.k, pr.v, pr.cu_seqlens, Hq=s.Hq, Hkv=s.Hkv, d=s.d, block=s.B,
                           dtype=pr.dtype, max_seqlen_q=max(s.lens_q), max_seqlen_k=max(s.lens_k),
                           seqlens_k=inp.seqlens_k.to(dev),
                           cu_seqlens_k=None if inp.paged else inp.cu_seqlens_k.to(dev),
                           page_table=pr.page_table, page_size=64 if inp.paged else 0,
                           q_scale=pr.keep[2], k_scale=pr.keep[3], v_scale=pr.keep[4],
                           out_dtype=fp2.FP2_FP8_E4M3, out_scale=out_scale)
    assert pr2.out.dtype == torch.float8_e4m3fn
    pr2.prefill(tau)
    pr2.check()
    deq = (pr2.out.float().cpu() * scale_h[None, :, None]).double().numpy()
    for b in range(inp.num_seqs):
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        a, e = int(inp.cu_seqlens_q[b]), int(inp.cu_seqlens_q[b + 1])
        got = deq[a:e].reshape(ref.shape)
        assert np.isfinite(got).all()
        rel, mx = H.compare(got, ref)
        assert rel <= H.FP8_REL_L2, f"seq {b}: rel-L2 {rel:.3e}"
