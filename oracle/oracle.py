"""ctypes front end of the fp64 CPU oracle (``fp2_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use this module; the product library never
imports it, and it imports nothing from the product package.

Every function works on ONE sequence in fp64, on the dequantised inputs:
Q ``[Lq, Hq, d]``, K and V ``[Lk, Hkv, d]``, query ``t`` at absolute position
``Lk - Lq + t``.  The method steps follow the FlashPrefill V2 abstract
(instantaneous pattern discovery, max-based dynamic thresholding, mean
correction term) and the popular explainer's section 2.1 (V1 keeps the
selected key blocks; V2 adds the mean of the dropped tokens); the readings
taken where those pages are silent are listed at the top of ``fp2_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp2_oracle.c")
_LIBS: dict[int, ctypes.CDLL] = {}
_LOCK = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)
_U8 = ctypes.POINTER(ctypes.c_ubyte)


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mut{mutant}.so"
    return os.path.join(_HERE, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc (``-O2 -fopenmp``); ``mutant`` > 0 builds a
    deliberately wrong variant for the mutation tests."""
    out = lib_path(mutant)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               f"-DFP2_ORACLE_MUTANT={mutant}", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, out)
    return out


def _lib(mutant: int = 0) -> ctypes.CDLL:
    with _LOCK:
        if mutant not in _LIBS:
            lib = ctypes.CDLL(build(mutant))
            lib.oracle_blockmean.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _D, _D, _I]
            lib.oracle_pool_q.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _D]
            lib.oracle_score.argtypes = [_D, _D] + [ctypes.c_int] * 6 + [_D]
            lib.oracle_mask.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, _U8]
            lib.oracle_attn_rows.argtypes = [_D, _D, _D, _D, _D, _I, _U8] + [ctypes.c_int] * 6 + \
                [_I, _I, ctypes.c_int, _D, _D]
            lib.oracle_dense_rows.argtypes = [_D, _D, _D] + [ctypes.c_int] * 5 + \
                [_I, _I, ctypes.c_int, _D]
            lib.oracle_num_threads.restype = ctypes.c_int
            _LIBS[mutant] = lib
        return _LIBS[mutant]


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def blockmean(K, V, B: int, mutant: int = 0):
    """Per-block means of K and V: ``kbar, vbar [Hkv, nkb, d]``, ``cnt [nkb]``."""
    K, V = _f64(K), _f64(V)
    Lk, Hkv, d = K.shape
    nkb = -(-Lk // B)
    kbar = np.zeros((Hkv, nkb, d)); vbar = np.zeros((Hkv, nkb, d))
    cnt = np.zeros(nkb, dtype=np.int32)
    _lib(mutant).oracle_blockmean(_p(K, _D), _p(V, _D), Lk, Hkv, d, B,
                                  _p(kbar, _D), _p(vbar, _D), _p(cnt, _I))
    return kbar, vbar, cnt


def pool_q(Q, B: int, off: int = 0, mutant: int = 0):
    """Pooled query blocks ``qbar [Hq, nqb, d]`` (mean over the valid rows);
    ``off`` = prefix mod B, the offset of row 0 inside its block."""
    Q = _f64(Q)
    Lq, Hq, d = Q.shape
    nqb = -(-(off + Lq) // B)
    qbar = np.zeros((Hq, nqb, d))
    _lib(mutant).oracle_pool_q(_p(Q, _D), Lq, Hq, d, B, off, _p(qbar, _D))
    return qbar


def score(qbar, kbar, prefix_blocks: int, mutant: int = 0):
    """Block scores ``S [Hq, nqb, nkb]``; entries with ``j > i_abs`` are NaN."""
    qbar, kbar = _f64(qbar), _f64(kbar)
    Hq, nqb, d = qbar.shape
    Hkv, nkb, _ = kbar.shape
    S = np.full((Hq, nqb, nkb), np.nan)
    _lib(mutant).oracle_score(_p(qbar, _D), _p(kbar, _D), Hq, Hkv, nqb, nkb, d, prefix_blocks,
                              _p(S, _D))
    return S


def mask(S, prefix_blocks: int, tau: float, mutant: int = 0):
    """Kept-block mask ``[Hq, nqb, nkb]`` (uint8, 1 = kept)."""
    S = _f64(S)
    Hq, nqb, nkb = S.shape
    keep = np.zeros((Hq, nqb, nkb), dtype=np.uint8)
    _lib(mutant).oracle_mask(_p(S, _D), Hq, nqb, nkb, prefix_blocks, float(tau), _p(keep, _U8))
    return keep


def attn_rows(Q, K, V, kbar, vbar, cnt, keep, B: int, rows, heads, want_wsum=False,
              mutant: int = 0):
    """Output rows ``[n, d]`` for the (row, head) pairs; optionally the sum of the
    normalised weights of every row (kept tokens + dropped-block pseudo-tokens)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    kbar, vbar = _f64(kbar), _f64(vbar)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    Lq, Hq, d = Q.shape
    Lk, Hkv, _ = K.shape
    n = rows.shape[0]
    out = np.zeros((n, d))
    wsum = np.zeros(n) if want_wsum else None
    _lib(mutant).oracle_attn_rows(_p(Q, _D), _p(K, _D), _p(V, _D), _p(kbar, _D), _p(vbar, _D),
                                  _p(cnt, _I), _p(keep, _U8), Lq, Lk, Hq, Hkv, d, B,
                                  _p(rows, _I), _p(heads, _I), n, _p(out, _D),
                                  _p(wsum, _D) if want_wsum else None)
    return (out, wsum) if want_wsum else out


def dense_rows(Q, K, V, rows, heads, mutant: int = 0):
    """Brute-force causal softmax(QK^T/sqrt(d))V for the (row, head) pairs."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    Lq, Hq, d = Q.shape
    Lk, Hkv, _ = K.shape
    n = rows.shape[0]
    out = np.zeros((n, d))
    _lib(mutant).oracle_dense_rows(_p(Q, _D), _p(K, _D), _p(V, _D), Lq, Lk, Hq, Hkv, d,
                                   _p(rows, _I), _p(heads, _I), n, _p(out, _D))
    return out


def dense_query_block(Qblk, K, V, p0: int, heads=None):
    """Causal softmax(QK^T/sqrt(d))V for a block of consecutive query rows, the
    first at absolute position ``p0`` (row r sees keys ``0 .. p0 + r``), with
    numpy fp64 matrix products as the steps (the same arithmetic as
    ``dense_rows``, in the order a matrix product takes): the method with
    every block kept (tau = +inf) is this dense causal attention, and the
    product form lets a long sequence be checked block by block.
    ``Qblk`` [n, Hq, d], ``K``/``V`` [>= p0 + n, Hkv, d]; returns
    [n * len(heads), d] ordered (row, head), like ``attn_query_block``."""
    Qblk = _f64(Qblk)
    n, Hq, d = Qblk.shape
    Hkv = np.asarray(K).shape[1]
    G = Hq // Hkv
    if heads is None:
        heads = np.arange(Hq, dtype=np.int32)
    heads = np.asarray(heads, dtype=np.int32)
    Lk = p0 + n
    Kd = _f64(np.asarray(K)[:Lk])
    Vd = _f64(np.asarray(V)[:Lk])
    # key t is visible to row r iff t <= p0 + r: only the last n keys can be
    # hidden from a row
    hidden = np.arange(n)[None, :] > np.arange(n)[:, None]
    out = np.empty((n, heads.size, d))
    for c, h in enumerate(heads):
        hk = h // G
        z = Qblk[:, h, :] @ Kd[:, hk, :].T
        z /= np.sqrt(d)
        z[:, p0:][hidden] = -np.inf
        z -= z.max(axis=1, keepdims=True)
        np.exp(z, out=z)
        out[:, c, :] = (z @ Vd[:, hk, :]) / z.sum(axis=1, keepdims=True)
    return out.reshape(n * heads.size, d)


def all_rows(Lq: int, Hq: int):
    """(rows, heads) covering every query row of every head."""
    t = np.repeat(np.arange(Lq, dtype=np.int32), Hq)
    h = np.tile(np.arange(Hq, dtype=np.int32), Lq)
    return t, h


class SeqResult:
    """Every intermediate of one sequence, as the oracle computes it."""

    def __init__(self, kbar, vbar, cnt, S, keep, out, rows, heads):
        self.kbar, self.vbar, self.cnt, self.S, self.keep = kbar, vbar, cnt, S, keep
        self.out, self.rows, self.heads = out, rows, heads


def group_pool(qbar, Hkv: int):
    """Group-shared masks (a variant): the pooled query of a KV group is the
    mean of its G heads' pooled queries, [Hkv, nqb, d]."""
    Hq, nqb, d = qbar.shape
    return np.asarray(qbar).reshape(Hkv, Hq // Hkv, nqb, d).mean(axis=1)


def prefill_seq(Q, K, V, B: int, tau: float, rows=None, heads=None, keep=None,
                group_masks: bool = False, mutant: int = 0) -> SeqResult:
    """All steps for one sequence: block means, pooled scores, threshold mask
    (unless ``keep`` is given), then the corrected sparse attention on the
    requested (row, head) pairs (all of them by default).  With
    ``group_masks`` every head of a KV group takes the group's mask, scored
    with the group-mean pooled query; ``S`` then holds the group score in
    each head's row."""
    Lq, Hq, _ = np.shape(Q)
    Lk = np.shape(K)[0]
    P = Lk - Lq
    if P < 0:
        raise ValueError("more queries than keys")
    kbar, vbar, cnt = blockmean(K, V, B, mutant)
    qbar = pool_q(Q, B, P % B, mutant)
    if group_masks:
        Hkv = kbar.shape[0]
        Sg = score(group_pool(qbar, Hkv), kbar, P // B, mutant)
        S = np.repeat(Sg, Hq // Hkv, axis=0)
    else:
        S = score(qbar, kbar, P // B, mutant)
    if keep is None:
        keep = mask(S, P // B, tau, mutant)
    if rows is None:
        rows, heads = all_rows(Lq, Hq)
    out = attn_rows(Q, K, V, kbar, vbar, cnt, keep, B, rows, heads, mutant=mutant)
    return SeqResult(kbar, vbar, cnt, S, keep, out, rows, heads)


# ---------------------------------------------------------------------------
# tau for a target drop fraction (harness reading: the pages give the target
# sparsities -- 70-85 % -- but not how tau is set; tau is put at the midpoint
# between the two adjacent margins m_i - s_ij at the target quantile, with one
# global tau per run).
# ---------------------------------------------------------------------------

def margins(S_list, prefix_blocks_list):
    """Margins ``m_i - s_ij`` of every causal, non-forced pair (0 < j < i_abs),
    and the number of causal pairs (forced ones included)."""
    ms = []
    total = 0
    for S, pb in zip(S_list, prefix_blocks_list):
        Hq, nqb, nkb = S.shape
        for i in range(nqb):
            iabs = pb + i
            row = S[:, i, : iabs + 1]
            m = row.max(axis=1, keepdims=True)
            total += Hq * (iabs + 1)
            if iabs >= 2:
                ms.append((m - row[:, 1:iabs]).ravel())
    return (np.concatenate(ms) if ms else np.zeros(0)), total


def tau_for_drop(S_list, prefix_blocks_list, target: float, guard: float = 0.0):
    """Global tau that drops ``target`` of all causal pairs.  With ``guard`` > 0
    the tau is moved to the nearest gap between adjacent margins that is wider
    than ``2*guard``, so that no score lies within ``guard`` of the threshold."""
    mg, total = margins(S_list, prefix_blocks_list)
    if mg.size == 0:
        return float("inf")
    a = np.sort(mg)
    n = a.size
    want = int(round(target * total))
    want = max(0, min(want, n))  # number of margins that must exceed tau
    if want == 0:
        return float(a[-1]) + 1.0
    if want == n:
        return float(a[0]) / 2.0 if a[0] > 0 else float(a[0]) - 1.0
    k = n - want  # tau between a[k-1] and a[k]
    if guard <= 0.0:
        return 0.5 * (float(a[k - 1]) + float(a[k]))
    gaps = a[1:] - a[:-1]
    ok = np.nonzero(gaps > 2.0 * guard)[0]
    if ok.size == 0:
        raise ValueError("no gap wide enough for the guard")
    best = ok[np.argmin(np.abs(ok - (k - 1)))]
    return 0.5 * (float(a[best]) + float(a[best + 1]))


def attn_query_block(Qblk, K, V, kbar, vbar, cnt, keep_i, B: int, iabs: int, heads=None,
                     p0: int | None = None, mutant: int = 0):
    """Corrected attention of ONE query block at absolute block index ``iabs``.

    ``Qblk`` [n, Hq, d] holds the block's rows, the first at absolute position
    ``p0`` (default ``iabs*B``; later for the partial first block of a call
    whose prefix is not a multiple of B), ``keep_i`` [Hq, >= iabs+1] its mask
    row.  Calls ``attn_rows`` on the causal window: keys ``[0, p0+n)`` (later
    keys never reach these rows) with the block as the whole query side, so
    that prefix = p0 puts every row at its true position.  No arithmetic of
    its own; it lets a long sequence be checked block by block without an
    fp64 copy of all of Q.  Returns [n * len(heads), d] ordered (row, head)."""
    Qblk = _f64(Qblk)
    n, Hq, d = Qblk.shape
    if p0 is None:
        p0 = iabs * B
    if p0 // B != iabs or (p0 + n - 1) // B != iabs:
        raise ValueError("the rows must lie in block iabs")
    Lk = p0 + n
    nkb = iabs + 1
    if heads is None:
        heads = np.arange(Hq, dtype=np.int32)
    heads = np.asarray(heads, dtype=np.int32)
    rows = np.repeat(np.arange(n, dtype=np.int32), heads.size)
    hh = np.tile(heads, n)
    keep = np.ascontiguousarray(np.asarray(keep_i)[:, None, :nkb], dtype=np.uint8)
    return attn_rows(Qblk, np.asarray(K)[:Lk], np.asarray(V)[:Lk], np.asarray(kbar)[:, :nkb],
                     np.asarray(vbar)[:, :nkb], np.asarray(cnt)[:nkb], keep, B, rows, hh,
                     mutant=mutant)
