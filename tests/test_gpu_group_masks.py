"""Group-shared masks (fp2_params.group_masks = 1, a variant of the method):
one kept set per KV group, scored with the group-mean pooled query.  The GPU
masks must equal the oracle's group masks bit for bit (tau placed in a gap of
the margins), be identical across the G heads of a group, and the outputs
must match the oracle run with those masks.  The distance to the per-head
method (the oracle's per-head output) is reported, not bounded."""
import numpy as np
import pytest

from block_sparse_long_blockmean_b200 import synth
from oracle import oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu

CASES = {
    "ragged_2k_g4": dict(lens_q=[2125], Hq=8, Hkv=2),
    "varlen_paged_g8_fp8": dict(lens_q=[700, 300], lens_k=[1024 + 700, 300], Hq=16, Hkv=2,
                                page_size=64, dtype="fp8"),
    "tiny_g4_d64_b64": dict(lens_q=[1024], Hq=4, Hkv=1, d=64, B=64, latents="per_block"),
    # G x block = 128: the two tiles of a CTA are adjacent query blocks
    "g2_b64_pairs_of_blocks": dict(lens_q=[1000, 1], lens_k=[1000, 777], Hq=4, Hkv=2, B=64),
    "g1_mha_unaligned": dict(lens_q=[300, 90], lens_k=[300 + 61, 90], Hq=4, Hkv=4),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_group_masks_match_oracle(name):
    inp = synth.make_inputs(H.small_shape(**CASES[name]))
    s = inp.shape
    G = s.Hq // s.Hkv
    res = []
    for b in range(inp.num_seqs):
        Q, K, V = inp.seq_q(b), inp.seq_k(b), inp.seq_v(b)
        res.append(O.prefill_seq(Q, K, V, s.B, np.inf, group_masks=True))
    pbs = [(s.lens_k[b] - s.lens_q[b]) // s.B for b in range(inp.num_seqs)]
    tau = O.tau_for_drop([r.S for r in res], pbs, 0.7, guard=1e-3)
    pr = H.problem(inp, out_fill=float("nan"), group_masks=True)
    pr.prefill(tau)
    pr.check()
    bits = H.gpu_bits(pr, inp)
    worst = 0.0
    for b in range(inp.num_seqs):
        Q, K, V = inp.seq_q(b), inp.seq_k(b), inp.seq_v(b)
        r = O.prefill_seq(Q, K, V, s.B, tau, group_masks=True)
        nqb, nkb = r.keep.shape[1:]
        assert (bits[b, :, :nqb, :nkb] == r.keep.astype(bool)).all()
        g = bits[b, :, :nqb, :nkb].reshape(s.Hkv, G, nqb, nkb)
        assert (g == g[:, :1]).all()
        got = H.out_seq(pr, inp, b).reshape(r.out.shape[0] // s.Hq, s.Hq, s.d)
        H.assert_close(got.reshape(r.out.shape), r.out, s.dtype == "fp8", f"{name} seq {b}")
        head = O.prefill_seq(Q, K, V, s.B, tau)
        worst = max(worst, H.compare(r.out, head.out)[0])
    print(f"{name}: group-mask vs per-head-mask output, oracle rel-L2 {worst:.3e}")
