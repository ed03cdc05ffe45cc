"""The contiguous workloads through an identity page table (pages in order,
64 tokens each): the paged path reads the same rows through the page table,
so block means, scores, masks and outputs must equal the contiguous run's bit
for bit, at the tiny, 32K and 128K sizes."""
import pytest
import torch

from block_sparse_long_blockmean_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cid", [1, 2, 3])
def test_identity_pages_equal_contiguous(cid):
    shape = synth.workload(cid, "bf16")
    contiguous = synth.make_inputs(shape, layout="contiguous")
    paged = synth.make_inputs(shape, layout="identity")
    assert torch.equal(contiguous.q, paged.q)
    tau = 2.5  # any finite tau: both runs take the same decisions
    a = H.problem(contiguous, out_fill=float("nan"), ws_fill=0)
    a.prefill(tau)
    a.check()
    b = H.problem(paged, out_fill=float("nan"), ws_fill=0)
    b.prefill(tau)
    b.check()
    L = a.layout()
    for name in ("kbar", "vbar", "scores", "kept_bits"):
        dt = torch.int32 if name == "kept_bits" else torch.float32
        last = L.nw if name == "kept_bits" else (shape.d if name in ("kbar", "vbar") else L.nkb_max)
        mid = (shape.Hkv, L.nkb_max) if name in ("kbar", "vbar") else (shape.Hq, L.nqb_max)
        x = a.ws_view(name, dt, (len(shape.lens_q), *mid, last))
        y = b.ws_view(name, dt, (len(shape.lens_q), *mid, last))
        assert torch.equal(x, y), name
    assert torch.equal(a.out, b.out)
    assert not torch.isnan(a.out.float()).any()
