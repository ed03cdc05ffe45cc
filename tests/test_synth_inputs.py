"""The seeded input generator (block_sparse_long_blockmean_b200/synth.py)
against its stated recipe: a latent per key block shared by the query and key
rows at the same absolute positions (q, k = 1.5 c_z + N(0, 1)), the first 4
key rows of each sequence x3 (sink), V ~ N(0, 1), bf16 rounding or e4m3
quantisation with per-head absmax/448 scales, and a paged cache whose page
table holds a seeded permutation of all pages.  Both the CUDA path and the
oracle read these inputs, so the checks here are on the generator alone."""
import numpy as np
import pytest
import torch

from block_sparse_long_blockmean_b200 import synth
from tests import harness as H


def _pooled(x, B):
    """[L, H, d] -> per-block means [H, nblk, d] (full blocks only)."""
    n = x.shape[0] // B
    return x[: n * B].reshape(n, B, x.shape[1], x.shape[2]).mean(axis=1).transpose(1, 0, 2)


def _cos(a, b):
    return (a * b).sum(-1) / np.linalg.norm(a, axis=-1) / np.linalg.norm(b, axis=-1)


@pytest.mark.parametrize("dtype,layout", [("bf16", "contiguous"), ("fp8", "paged")])
def test_same_seed_same_inputs(dtype, layout):
    shape = H.small_shape([300, 40], [500, 40], Hq=4, Hkv=2, d=64, B=64, dtype=dtype,
                          page_size=32 if layout == "paged" else 0, seed=5)
    a, b = synth.make_inputs(shape), synth.make_inputs(shape)
    for x, y in [(a.q, b.q), (a.k, b.k), (a.v, b.v)]:
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    if layout == "paged":
        assert torch.equal(a.page_table, b.page_table)
    other = synth.make_inputs(H.small_shape([300, 40], [500, 40], Hq=4, Hkv=2, d=64, B=64,
                                            dtype=dtype, seed=6))
    assert not torch.equal(a.q.view(torch.uint8), other.q.view(torch.uint8))


@pytest.mark.parametrize("layout", ["paged", "identity"])
def test_page_table_and_cache(layout):
    lens_k = [130, 64, 1, 257]
    shape = H.small_shape([30, 64, 1, 100], lens_k, Hq=4, Hkv=2, d=64, B=64, page_size=32,
                          seed=8)
    inp = synth.make_inputs(shape, layout)
    ps = inp.k.shape[1]
    npages = [-(-L // ps) for L in lens_k]
    table = inp.page_table.numpy()
    used = np.concatenate([table[b, :n] for b, n in enumerate(npages)])
    assert sorted(used.tolist()) == list(range(sum(npages)))   # every page exactly once
    if layout == "identity":
        assert used.tolist() == list(range(sum(npages)))
    else:
        assert used.tolist() != sorted(used.tolist())             # permuted
    for b, n in enumerate(npages):
        assert (table[b, n:] == -1).all()
    # gathering through the table gives back the contiguous rows; page tails are zero
    cu = inp.cu_seqlens_k.numpy()
    for b, L in enumerate(lens_k):
        for t in range(L):
            pg, r = table[b, t // ps], t % ps
            assert torch.equal(inp.k[pg, r], inp._kc[cu[b] + t])
            assert torch.equal(inp.v[pg, r], inp._vc[cu[b] + t])
        last = table[b, npages[b] - 1]
        tail = L - (npages[b] - 1) * ps
        assert not inp.k[last, tail:].float().any() and not inp.v[last, tail:].float().any()


def test_fp8_scales_are_per_head_absmax():
    shape = H.small_shape([200], [200], Hq=4, Hkv=2, d=64, B=64, dtype="fp8", seed=9)
    inp = synth.make_inputs(shape)
    for x, sc, H_ in [(inp.q, inp.q_scale, 4), (inp._kc, inp.k_scale, 2), (inp._vc, inp.v_scale, 2)]:
        assert x.dtype == torch.float8_e4m3fn and sc.shape == (H_,)
        amax = x.float().abs().amax(dim=(0, 2))
        # each head's largest value lands on the format's largest finite value
        assert torch.equal(amax, torch.full((H_,), synth.E4M3_MAX))
        assert (sc > 0).all()


def test_latents_sink_and_values():
    """Per-block latents (the tiny workload's recipe): a query block's pooled
    query points the same way as its own key block's mean and not the
    others'; the first 4 key rows are ~3x longer; V is unit-variance noise."""
    shape = synth.workload(1)
    inp = synth.make_inputs(shape)
    B = shape.B
    q, k, v = inp.seq_q(0), inp.seq_k(0), inp.seq_v(0)
    G = shape.Hq // shape.Hkv
    qb = _pooled(q, B)                                   # [Hq, n, d]
    kb = _pooled(k, B)                                   # [Hkv, n, d]
    for h in range(shape.Hq):
        cos = _cos(qb[h][:, None, :], kb[h // G][None, :, :])   # [n, n]
        n = cos.shape[0]
        diag = np.diag(cos)
        off = cos[~np.eye(n, dtype=bool)]
        assert diag.min() > 0.8 and np.abs(off).mean() < 0.2
    norms = np.linalg.norm(k, axis=-1)                  # [L, Hkv]
    ratio = norms[:4].mean() / norms[4:B].mean()
    assert 2.5 < ratio < 3.5
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.02


def test_query_latents_follow_absolute_positions():
    """With a prefix that is not a multiple of the block, a query row takes
    the latent of the key block at its absolute position."""
    B, P, Lq = 64, 100, 300
    shape = H.small_shape([Lq], [P + Lq], Hq=2, Hkv=2, d=64, B=B, latents="per_block", seed=12)
    inp = synth.make_inputs(shape)
    q, k = inp.seq_q(0), inp.seq_k(0)
    kb = _pooled(k, B)                                  # key blocks 0..5 (full ones)
    for j in range(P // B + 1, (P + Lq) // B):          # absolute blocks wholly in the call
        rows = q[j * B - P:(j + 1) * B - P].mean(axis=0)  # [Hq, d]
        cos = _cos(rows[:, None, :], kb)                  # [Hq, nkb] (Hq = Hkv here)
        assert (cos.argmax(axis=1) == j).all()


def test_workload_sizes():
    w4 = synth.workload(4)
    assert len(w4.lens_q) == 8 and w4.lens_q == w4.lens_k
    assert all(4096 <= L <= 65536 for L in w4.lens_q)
    assert (w4.page_size, w4.dtype, w4.Hq, w4.Hkv, w4.d, w4.B) == (64, "fp8", 32, 8, 128, 128)
    w5 = synth.workload(5)
    assert (w5.lens_q, w5.lens_k, w5.Hq, w5.page_size, w5.dtype) == ([32768], [262144], 64, 64,
                                                                      "fp8")
    w3 = synth.workload(3)
    assert (w3.lens_q, w3.Hq, w3.Hkv, w3.d, w3.B, w3.drop) == ([131072], 32, 8, 128, 128, 0.8)
    for cid in range(1, 6):
        assert synth.workload(cid).seed == 20260822 + cid
