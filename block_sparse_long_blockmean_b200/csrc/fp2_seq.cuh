// fp2_seq.cuh -- per-sequence bookkeeping shared by the fp2 kernels: where a
// call's query rows sit among the key blocks when the call is a chunk on a
// resident prefix, of any length (FlashPrefill V2 popular explainer, section
// 2.3 system layer: chunked prefill, chunks that mix prefill and decode rows).
#pragma once

#include "fp2_device.cuh"
#include "fp2_internal.h"

namespace fp2 {

struct SeqInfo {
    int q0;  // first row of the sequence in q / out
    int Lq;  // new (query) tokens
    int k0;  // first row in contiguous K/V (0 when paged)
    int Lk;  // keys (resident prefix + new tokens)
    int P;   // prefix length Lk - Lq; query t sits at absolute position P + t
    // Query blocks are cut at absolute positions: query block i of the call
    // is absolute block pb + i and holds the rows t with (P + t) / B == pb + i.
    // When P is not a multiple of B (a decode row, a chunk that ends inside a
    // block) the first one starts `off` rows into its block and is partial.
    int pb;   // P / B
    int off;  // P % B
    int nqb;  // query blocks of the call: ceil((off + Lq) / B), 0 when Lq = 0
};

// Reads sequence b's lengths and checks them against the launch's limits.
// On a violation it records the error (once per grid, first writer wins) and
// returns false; the caller then skips its work.
__device__ __forceinline__ bool load_seq(const KParams& p, int b, SeqInfo& s) {
    s.q0 = p.cu_q[b];
    s.Lq = p.cu_q[b + 1] - s.q0;
    s.Lk = p.seqlens_k ? p.seqlens_k[b] : s.Lq;
    s.k0 = p.paged ? 0 : p.cu_k[b];
    s.P = s.Lk - s.Lq;
    const bool lens_ok = s.Lq >= 0 && s.Lq <= p.max_seqlen_q && s.Lk <= p.max_seqlen_k &&
                         s.P >= 0 && s.q0 >= 0 && s.q0 + s.Lq <= p.total_q;
    const bool keys_ok = !p.uses_kv ? true : p.paged ? (s.Lk + p.page_size - 1) / p.page_size <= p.max_pages
                                 : (s.k0 >= 0 && s.k0 + s.Lk <= p.total_k);
    if (!lens_ok || !keys_ok) {
        set_error(p.err, lens_ok ? kErrBounds : kErrInvalid, kDetSeqLen);
        return false;
    }
    s.pb = s.P / p.B;
    s.off = s.P - s.pb * p.B;
    s.nqb = s.Lq > 0 ? (s.off + s.Lq + p.B - 1) / p.B : 0;
    return true;
}

// Row index (in units of Hkv*d elements) of key token `tok` of sequence b,
// or -1 (error recorded) when its page id is out of range.
__device__ __forceinline__ long long key_row(const KParams& p, const SeqInfo& s, int b, int tok) {
    if (!p.paged) return (long long)s.k0 + tok;
    const int pg = p.page_table[(size_t)b * p.max_pages + tok / p.page_size];
    if (pg < 0 || pg >= p.num_pages) {
        set_error(p.err, kErrBounds, kDetPage);
        return -1;
    }
    return (long long)pg * p.page_size + (tok % p.page_size);
}

}  // namespace fp2
