"""The bounded-wait error path of the attention kernel, made to run out on
purpose without faulting anything: a test-only knob (fp2_params
debug_withhold_k_item) makes the producer never load one K tile, and a short
wait limit (debug_wait_limit_us) makes the consumer waiting for it give up.
The call must report FP2_ERR_TIMEOUT through the workspace error word, leave
the context usable, and the next normal call on the same workspace must be
correct (the aborted CTAs drained their copies and MMAs and freed TMEM)."""
import numpy as np
import pytest

from block_sparse_long_blockmean_b200 import fp2, synth
from oracle import oracle as O
from tests import harness as H

WAIT_DETAIL_BASE = 16  # detail codes of pipeline wait sites start here


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,page", [("bf16", 0), ("fp8", 64)])
def test_withheld_tile_times_out_then_next_call_is_correct(dtype, page):
    shape = H.small_shape([640, 384], Hq=8, Hkv=2, dtype=dtype, page_size=page, seed=31)
    inp = synth.make_inputs(shape)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.4)
    pr = H.problem(inp, out_fill=float("nan"))
    # every CTA whose work list reaches item 2 waits for a K tile that never comes
    pr.params.debug_wait_limit_us = 20000
    pr.params.debug_withhold_k_item = 2
    pr.prefill(tau)
    st, det = fp2.get_status(pr.params)
    assert st == fp2.FP2_ERR_TIMEOUT, fp2.status_string(st)
    assert WAIT_DETAIL_BASE <= det < WAIT_DETAIL_BASE + 16, det
    # reading the status cleared it
    assert fp2.get_status(pr.params) == (fp2.FP2_OK, 0)

    pr.params.debug_wait_limit_us = 0
    pr.params.debug_withhold_k_item = 0
    pr.out.fill_(float("nan"))
    pr.prefill(tau)
    pr.check()
    for b in range(inp.num_seqs):
        keep = O.mask(orc[b][3], orc[b][4], tau)
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        got = H.out_seq(pr, inp, b).reshape(ref.shape)
        assert np.isfinite(got).all()
        H.assert_close(got, ref, dtype == "fp8", f"seq {b} after the timed-out call")


def test_debug_knobs_are_validated_on_the_host():
    """A negative item index is an argument error, caught before any launch."""
    P = fp2.Params()
    P.num_seqs, P.num_q_heads, P.num_kv_heads, P.head_dim = 1, 8, 2, 128
    P.total_q = P.total_k = P.max_seqlen_q = P.max_seqlen_k = 256
    P.debug_withhold_k_item = -1
    assert fp2.workspace_size(P, 128) == 0
    P.debug_withhold_k_item = 0
    P.attn_kernel = 2
    assert fp2.workspace_size(P, 128) == 0
    P.attn_kernel = 1
    assert fp2.workspace_size(P, 128) > 0
