"""fp2_prefill_host: q, K/V and out in pinned host memory, copies pipelined
with the kernels over query-block chunks on three streams.  Its output must
be bit-identical to fp2_prefill on the same data already on the device, for
any chunk count, and two calls queued back to back on the same device
buffers (different inputs, no synchronisation between them) must each give
their own result."""
import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import fp2, synth
from tests import harness as H

pytestmark = pytest.mark.gpu

SHAPES = {
    "single_4k_bf16": dict(lens_q=[4000], Hq=8, Hkv=2),
    "mixed_paged_fp8": dict(lens_q=[1, 37, 700, 0, 300], lens_k=[3001, 1000, 1713, 64, 300],
                            Hq=8, Hkv=2, page_size=64, dtype="fp8"),
    "chunk_g8_b64": dict(lens_q=[900, 5], lens_k=[900 + 333, 1000], Hq=16, Hkv=2, B=64,
                         page_size=32),
    "mixed_contiguous": dict(lens_q=[1, 600, 0, 250, 1], lens_k=[2500, 600, 300, 1900, 129],
                             Hq=8, Hkv=2),
}


def device_reference(inp, tau, out_dtype=fp2.FP2_BF16):
    pr = H.problem(inp, out_fill=float("nan"))
    if out_dtype != fp2.FP2_BF16:
        pr.params.out_dtype = out_dtype
        pr.out = torch.zeros(pr.out.shape, dtype=torch.uint8, device="cuda")
    pr.prefill(tau)
    pr.check()
    return pr


def host_call(pr, inp, tau, num_chunks, streams, out_host):
    # the device buffers start as NaN bytes: every row the kernels read must
    # have been uploaded by the call itself
    for t in (pr.q, pr.k, pr.v, pr.out):
        t.view(torch.uint8).fill_(0xFF)
    hq = inp.q.pin_memory()
    hk = inp.k.pin_memory()
    hv = inp.v.pin_memory()
    cu_h = inp.cu_seqlens_q.to(torch.int32).contiguous()
    lk_h = inp.seqlens_k.to(torch.int32).contiguous()
    cuk_h = None if inp.paged else inp.cu_seqlens_k.to(torch.int32).contiguous()
    io = fp2.host_io(hq, hk, hv, out_host, pr.q, pr.k, pr.v, pr.out, cu_h, lk_h,
                     upload_stream=streams[0], download_stream=streams[1],
                     num_chunks=num_chunks, cu_seqlens_k_host=cuk_h)
    fp2.prefill_host(io, pr.page_table, pr.cu_seqlens, tau, inp.shape.B, pr.dtype, pr.params)
    return (hq, hk, hv, cu_h, lk_h, cuk_h)  # keep alive until the stream is synchronised


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("num_chunks", [1, 3, 16, 64])
def test_host_path_matches_device_path(name, num_chunks):
    inp = synth.make_inputs(H.small_shape(**SHAPES[name], seed=61))
    tau = H.pick_tau(H.oracle_scores(inp), 0.6)
    ref = device_reference(inp, tau)
    pr = H.problem(inp, out_fill=float("nan"))
    out_host = torch.full(pr.out.shape, float("nan"), dtype=pr.out.dtype).pin_memory()
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    keep = host_call(pr, inp, tau, num_chunks, streams, out_host)
    torch.cuda.current_stream().synchronize()
    torch.cuda.synchronize()
    pr.check()
    del keep
    assert torch.equal(out_host, ref.out.cpu())


def test_back_to_back_calls_do_not_race():
    shape = dict(SHAPES["single_4k_bf16"])
    a = synth.make_inputs(H.small_shape(**shape, seed=62))
    b = synth.make_inputs(H.small_shape(**shape, seed=63))
    tau = H.pick_tau(H.oracle_scores(a), 0.6)
    ref_a, ref_b = device_reference(a, tau), device_reference(b, tau)
    assert not torch.equal(ref_a.out, ref_b.out)
    pr = H.problem(a, out_fill=float("nan"))
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    out_a = torch.empty(pr.out.shape, dtype=pr.out.dtype).pin_memory()
    out_b = torch.empty(pr.out.shape, dtype=pr.out.dtype).pin_memory()
    keep_a = host_call(pr, a, tau, 4, streams, out_a)
    keep_b = host_call(pr, b, tau, 4, streams, out_b)  # same device buffers, no sync between
    torch.cuda.synchronize()
    pr.check()
    del keep_a, keep_b
    assert torch.equal(out_a, ref_a.out.cpu())
    assert torch.equal(out_b, ref_b.out.cpu())


def test_e4m3_output_through_host_path():
    inp = synth.make_inputs(H.small_shape(**SHAPES["mixed_paged_fp8"], seed=64))
    tau = H.pick_tau(H.oracle_scores(inp), 0.6)
    ref = device_reference(inp, tau, out_dtype=fp2.FP2_FP8_E4M3)
    pr = H.problem(inp)
    pr.params.out_dtype = fp2.FP2_FP8_E4M3
    pr.out = torch.zeros(pr.out.shape, dtype=torch.uint8, device="cuda")
    out_host = torch.full(pr.out.shape, 0xFF, dtype=torch.uint8).pin_memory()
    keep = host_call(pr, inp, tau, 5, (torch.cuda.Stream(), torch.cuda.Stream()), out_host)
    torch.cuda.synchronize()
    pr.check()
    del keep
    assert torch.equal(out_host, ref.out.cpu())


def test_single_stream_when_no_copy_streams_are_given():
    inp = synth.make_inputs(H.small_shape(**SHAPES["chunk_g8_b64"], seed=65))
    tau = H.pick_tau(H.oracle_scores(inp), 0.6)
    ref = device_reference(inp, tau)
    pr = H.problem(inp, out_fill=float("nan"))
    out_host = torch.full(pr.out.shape, float("nan"), dtype=pr.out.dtype).pin_memory()
    keep = host_call(pr, inp, tau, 3, (None, None), out_host)
    torch.cuda.synchronize()
    del keep
    assert torch.equal(out_host, ref.out.cpu())
    assert np.isfinite(out_host.float().numpy()).all()


@pytest.mark.parametrize("page", [64, 0])
def test_block_scaled_cache_through_host_path(page):
    """An e4m3 cache quantised per key block (per-block factors stay device
    arrays, like the lengths): the host path equals the device path bit for bit."""
    kw = dict(lens_q=[700, 1, 300], lens_k=[700 + 256, 900, 300], Hq=8, Hkv=2, dtype="fp8",
              page_size=page, kv_scales="block")
    if not page:  # contiguous K/V carries no prefix
        kw["lens_k"] = list(kw["lens_q"])
    inp = synth.make_inputs(H.small_shape(**kw, seed=66))
    tau = H.pick_tau(H.oracle_scores(inp), 0.6)
    ref = device_reference(inp, tau)
    pr = H.problem(inp, out_fill=float("nan"))
    out_host = torch.full(pr.out.shape, float("nan"), dtype=pr.out.dtype).pin_memory()
    keep = host_call(pr, inp, tau, 4, (torch.cuda.Stream(), torch.cuda.Stream()), out_host)
    torch.cuda.synchronize()
    pr.check()
    del keep
    assert torch.equal(out_host, ref.out.cpu())
