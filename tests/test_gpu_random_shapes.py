"""GPU parity over a seeded sweep of small random problems: every supported
combination of head dim, block, GQA group, dtype and KV layout, batches that
mix fresh prefills, chunks on aligned and unaligned prefixes, decode rows and
empty sequences; both attention kernels (the one-tile kernel also forced on
problems the two-tile kernel would take).

Each problem is compared with the fp64 oracle: masks bit exact (tau sits in
a gap of the oracle's margins, no score within 1e-3 of the threshold) and
outputs within the bf16 / e4m3 tolerances of the other parity tests."""
import numpy as np
import pytest

from block_sparse_long_blockmean_b200 import synth
from oracle import oracle as O
from tests import harness as H

N_CASES = 24


def random_case(k: int):
    """Problem k of the sweep (deterministic): shape kwargs and whether the
    one-tile kernel is forced."""
    rng = np.random.default_rng(7000 + k)
    fp8 = rng.random() < 0.3
    d = 128 if fp8 else int(rng.choice([64, 128]))
    B = 128 if fp8 else int(rng.choice([64, 128]))  # e4m3 runs with d = block = 128
    G = int(rng.choice([g for g in (1, 2, 4, 8) if 128 // g <= B]))
    Hkv = int(rng.integers(1, 4))
    page_size = 0
    if rng.random() < 0.5:
        page_size = int(rng.choice([p for p in (16, 32, 64, 128, 256) if B % p == 0 or p % B == 0]))
    lens_q, lens_k = [], []
    for _ in range(int(rng.integers(1, 5))):
        kind = rng.choice(["prefill", "aligned", "unaligned", "decode", "empty"],
                          p=[0.3, 0.2, 0.25, 0.15, 0.1])
        if kind == "prefill":
            q = int(rng.integers(1, 600)); p = 0
        elif kind == "aligned":
            q = int(rng.integers(1, 500)); p = B * int(rng.integers(1, 1200 // B))
        elif kind == "unaligned":
            q = int(rng.integers(1, 500)); p = int(rng.integers(1, 1300))
        elif kind == "decode":
            q = 1; p = int(rng.integers(0, 1800))
        else:
            q = 0; p = int(rng.integers(0, 700))
        lens_q.append(q)
        lens_k.append(q + p)
    if max(lens_q) == 0:
        lens_q[0], lens_k[0] = 1, lens_k[0] + 1
    kw = dict(lens_q=lens_q, lens_k=lens_k, Hq=G * Hkv, Hkv=Hkv, d=d, B=B,
              dtype="fp8" if fp8 else "bf16", page_size=page_size,
              drop=float(rng.uniform(0.3, 0.8)), seed=9000 + k)
    force_single = G * B >= 256 and rng.random() < 0.3
    return kw, force_single


@pytest.mark.gpu
@pytest.mark.parametrize("k", range(N_CASES))
def test_random_problem(k):
    kw, force_single = random_case(k)
    inp = synth.make_inputs(H.small_shape(**kw))
    orc = H.oracle_scores(inp)
    tau = H.pick_tau(orc, kw["drop"])
    pr = H.problem(inp, out_fill=float("nan"), ws_fill=0xFF, attn_kernel=int(force_single))
    pr.prefill(tau)
    pr.check()
    got = H.gpu_bits(pr, inp)
    fp8 = kw["dtype"] == "fp8"
    for b in range(inp.num_seqs):
        S, pb = orc[b][3], orc[b][4]
        nqb, nkb = S.shape[1], S.shape[2]
        keep = O.mask(S, pb, tau)
        assert (got[b, :, :nqb, :nkb] == keep.astype(bool)).all(), f"case {k} seq {b}: mask"
        assert not got[b, :, :nqb, nkb:].any()
        if kw["lens_q"][b] == 0:
            continue
        ref, _, _ = H.oracle_out(inp, b, orc[b], keep)
        out = H.out_seq(pr, inp, b).reshape(ref.shape)
        assert np.isfinite(out).all(), f"case {k} seq {b}: non-finite output"
        H.assert_close(out, ref, fp8, f"case {k} {kw} single={force_single} seq {b}")


def test_sweep_covers_the_supported_space():
    """The sweep (a CPU check of the generator) reaches every kernel and
    layout it is meant to: both dtypes, d 64 and 128, blocks 64 and 128,
    every group size, paged and contiguous K/V, unaligned prefixes, decode
    rows, empty sequences and the forced one-tile kernel."""
    seen = set()
    for k in range(N_CASES):
        kw, single = random_case(k)
        seen.add(("dtype", kw["dtype"]))
        seen.add(("d", kw["d"]))
        seen.add(("B", kw["B"]))
        seen.add(("G", kw["Hq"] // kw["Hkv"]))
        seen.add(("paged", kw["page_size"] > 0))
        seen.add(("single", single))
        for q, kk in zip(kw["lens_q"], kw["lens_k"]):
            p = kk - q
            if q == 0:
                seen.add(("empty", True))
            elif q == 1 and p > 0:
                seen.add(("decode", True))
            elif p % kw["B"]:
                seen.add(("unaligned", True))
    want = {("dtype", "bf16"), ("dtype", "fp8"), ("d", 64), ("d", 128), ("B", 64), ("B", 128),
            ("G", 1), ("G", 2), ("G", 4), ("G", 8), ("paged", True), ("paged", False),
            ("single", True), ("single", False), ("empty", True), ("decode", True),
            ("unaligned", True)}
    assert want <= seen, want - seen
