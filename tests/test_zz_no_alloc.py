"""fp2_prefill_noalloc -- the prefill for callers that cannot allocate device
memory (plugin-style hosts that pass a kernel only its inputs and outputs,
runtimes that reserve all device memory up front) -- checked through the C ABI
against fp2_prefill on the same inputs, on two calls in a row.  This file is
collected last on purpose: it must pass alone in a fresh process and after
every other test."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from tests import harness as H


def _noalloc(pr, tau, block, out):
    return fp2.lib().fp2_prefill_noalloc(
        pr.q.data_ptr(), pr.k.data_ptr(), pr.v.data_ptr(),
        pr.page_table.data_ptr() if pr.page_table is not None else None,
        pr.cu_seqlens.data_ptr(), ctypes.c_float(tau), block, pr.dtype, out.data_ptr(),
        ctypes.byref(pr.params))


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,page", [("bf16", 64), ("fp8", 0)])
def test_noalloc_matches_prefill_on_two_calls(dtype, page):
    """Same four launches on the same inputs as fp2_prefill, so the output
    must be the same bits on both calls: stale scratch left by the first call
    (kept lists, mean tiles) would show up on the second."""
    shape = H.small_shape([700, 300], lens_k=[256 + 700, 300], Hq=8, Hkv=2, dtype=dtype,
                          page_size=page if page else 0, seed=23)
    if page == 0:  # contiguous K/V cannot carry a prefix
        shape.lens_k = list(shape.lens_q)
    inp = synth.make_inputs(shape)
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, 0.6)
    pr = H.problem(inp)
    pr.prefill(tau)
    pr.check()
    for call in range(2):
        out = torch.full_like(pr.out, float("nan"))
        st = _noalloc(pr, tau, shape.B, out)
        assert st == fp2.FP2_OK, fp2.status_string(st)
        torch.cuda.synchronize()
        assert fp2.noalloc_get_status() == (fp2.FP2_OK, 0), f"call {call}"
        assert np.isfinite(out.double().cpu().numpy()).all(), f"call {call}"
        assert torch.equal(out.view(torch.uint8), pr.out.view(torch.uint8)), f"call {call}"


@pytest.mark.gpu
def test_noalloc_reports_device_errors_and_clears_them():
    """A page id out of range (the kernels check it and skip the access) is
    recorded in the library-owned array and read back, then cleared."""
    inp = synth.make_inputs(H.small_shape([300, 200], Hq=8, Hkv=2, page_size=64, seed=5))
    pr = H.problem(inp)
    pt = pr.page_table.clone()
    pt[1, 0] = 10 ** 6
    pr.page_table = pt
    out = torch.empty_like(pr.out)
    assert _noalloc(pr, 1.0, 128, out) == fp2.FP2_OK
    assert fp2.noalloc_get_status() == (fp2.FP2_ERR_DEVICE_BOUNDS, 3)
    assert fp2.noalloc_get_status() == (fp2.FP2_OK, 0)


def test_noalloc_rejects_problems_above_its_scratch():
    """Rejected on the host before any device work (no GPU needed)."""
    P = fp2.Params()
    P.num_seqs, P.num_q_heads, P.num_kv_heads, P.head_dim = 1, 32, 8, 128
    P.total_q = P.total_k = P.max_seqlen_q = P.max_seqlen_k = 131072
    assert fp2.workspace_size(P, 128) > 32 * 1024 * 1024
    fake = 1 << 20
    st = fp2.lib().fp2_prefill_noalloc(fake, fake, fake, None, fake, ctypes.c_float(1.0), 128,
                                       fp2.FP2_BF16, fake, ctypes.byref(P))
    assert st == fp2.FP2_ERR_WORKSPACE


def test_noalloc_rejects_bad_arguments_before_touching_the_array():
    """A NaN tau or a misaligned output is an argument error, returned
    before anything is queued (no GPU needed: nothing reaches the device)."""
    P = fp2.Params()
    P.num_seqs, P.num_q_heads, P.num_kv_heads, P.head_dim = 1, 8, 2, 128
    P.total_q = P.total_k = P.max_seqlen_q = P.max_seqlen_k = 256
    fake = 1 << 20
    lib = fp2.lib()
    st = lib.fp2_prefill_noalloc(fake, fake, fake, None, fake, ctypes.c_float(float("nan")),
                                 128, fp2.FP2_BF16, fake, ctypes.byref(P))
    assert st == fp2.FP2_ERR_INVALID_ARG
    st = lib.fp2_prefill_noalloc(fake, fake, fake, None, fake, ctypes.c_float(1.0), 128,
                                 fp2.FP2_BF16, fake + 8, ctypes.byref(P))
    assert st == fp2.FP2_ERR_INVALID_ARG
