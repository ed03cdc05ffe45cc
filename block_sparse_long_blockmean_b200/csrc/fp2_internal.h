// fp2_internal.h -- parameter block shared by the host launcher and the
// kernels of the fp2 library (not part of the public ABI).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

namespace fp2 {

struct KParams {
    int num_seqs, Hq, Hkv, d, G, B;
    int total_q, total_k;
    int paged, page_size, max_pages, num_pages;
    int max_seqlen_q, max_seqlen_k;
    int nqb_max, nkb_max, nw;
    // query blocks [qb_lo, qb_lo + qb_n) of every sequence are processed by
    // the score, mask and attention launches (all of them: 0, nqb_max)
    int qb_lo, qb_n;
    // key blocks [kb_lo, kb_lo + kb_n) are averaged by the block-mean launch
    // (all of them: 0, nkb_max)
    int kb_lo, kb_n;
    int fp8;
    int uses_kv;               // 0: the launch never reads K/V (no key-extent check)
    int group_masks;           // score every head with its group's mean pooled query
    int out_fp8;               // e4m3 output (O / out_scale), else bf16
    const float* out_scale;    // [Hq] or nullptr (FP8 inputs: v_scale of the KV head)
    const int32_t* cu_q;       // [S+1]
    const int32_t* cu_k;       // [S+1] contiguous key offsets (may alias cu_q)
    const int32_t* seqlens_k;  // [S] or nullptr
    const int32_t* page_table; // [S][max_pages] or nullptr
    const float* q_scale;
    const float* k_scale;
    const float* v_scale;
    uint32_t* err;             // error word (workspace)
    float* kbar;               // [S][Hkv][nkb_max][d]
    float* vbar;
    void* kbar_op;             // bf16 | e4m3, same shape
    void* vbar_op;
    float* scores;             // [S][Hq][nqb_max][nkb_max]
    int32_t* kept_idx;         // [S][Hq][nqb_max][nkb_max]
    int32_t* kept_cnt;         // [S][Hq][nqb_max]
    uint32_t* kept_bits;       // [S][Hq][nqb_max][nw]
    // optional block-mean cache (chunked prefill): raw means of the stored
    // K and V values, [num_slots][2][Hkv][d] fp32, slot of (b, j) in
    // block_table[b * max_blocks + j]
    float* mean_cache;
    const int32_t* block_table;
    int max_blocks, num_slots;
    // limit of every pipeline wait of the attention kernels, in ns (0: the
    // default 2 s); test-only knob of the bounded-wait error path
    unsigned long long wait_limit_ns;
    // > 0: the attention producer withholds the K tile of that work item
    // (1-based) in every CTA, so the consumer's bounded wait runs out
    // (test-only; 0 in every normal call)
    int withhold_k_item;
    int attn_kernel;           // 0: two-tile kernel, 1: one-tile kernel
    // e4m3 only, optional: per-block scale factors in (0, 1] of K and V,
    // [S][nkb_max][Hkv] (x = e4m3 * k_scale[h] * factor), or nullptr
    const float* kb_fac;
    const float* vb_fac;
};

// Detail codes stored beside an error code.
enum : uint32_t {
    kDetSeqLen = 1,      // Lq or Lk outside [0, max_seqlen_*] or Lk < Lq
    kDetPage = 3,        // page id outside [0, num_pages)
    kDetSlot = 4,        // block-mean cache slot outside [0, num_slots) or beyond max_blocks
    kDetFactor = 5,      // a per-block scale factor outside (0, 1]
    kDetWaitBase = 16,   // + pipeline wait site
};

// Launchers (fp2_stages.cu, fp2_attn.cu).  Return the launch error.
cudaError_t launch_blockmean(const KParams& p, const void* k, const void* v, cudaStream_t s);
cudaError_t launch_score(const KParams& p, const void* q, cudaStream_t s);
cudaError_t launch_mask(const KParams& p, float tau, cudaStream_t s);
cudaError_t launch_attn(const KParams& p, const void* q, const void* k, const void* v,
                        const uint32_t* kept_bits, void* out, cudaStream_t s);

}  // namespace fp2
