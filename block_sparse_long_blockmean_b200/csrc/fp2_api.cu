// fp2_api.cu -- the C ABI of include/fp2.h: argument validation, workspace
// layout, stream-ordered launches of the four kernels, the host-buffer
// pipeline, status read-back and the host-side tau calibration utility.
// fp2_prefill runs the method's four steps in the order the FlashPrefill V2
// abstract gives them (block statistics, pattern discovery, dynamic
// threshold, sparse attention with the mean correction); the host-buffer
// pipeline and the tau utility are packaging with no counterpart there.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "fp2.h"
#include "fp2_internal.h"

using fp2::KParams;

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

fp2_status check_params(const fp2_params* P, int block) {
    if (!P) return FP2_ERR_INVALID_ARG;
    if (P->num_seqs < 1 || P->num_q_heads < 1 || P->num_kv_heads < 1 || P->total_q < 0 ||
        P->max_seqlen_q < 0 || P->max_seqlen_k < P->max_seqlen_q || P->max_seqlen_k < 1)
        return FP2_ERR_INVALID_ARG;
    if (P->num_q_heads % P->num_kv_heads != 0) return FP2_ERR_INVALID_ARG;
    if (P->attn_kernel != 0 && P->attn_kernel != 1) return FP2_ERR_INVALID_ARG;
    if (P->debug_withhold_k_item < 0) return FP2_ERR_INVALID_ARG;
    const int G = P->num_q_heads / P->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return FP2_ERR_UNSUPPORTED;
    if (P->head_dim != 64 && P->head_dim != 128) return FP2_ERR_UNSUPPORTED;
    if (block != 64 && block != 128) return FP2_ERR_UNSUPPORTED;
    if (128 / G > block) return FP2_ERR_UNSUPPORTED;
    return FP2_OK;
}

fp2_status check_kv(const fp2_params* P, int block, const int32_t* page_table) {
    if (page_table) {
        if (!is_pow2(P->page_size) || P->page_size < 16 || P->page_size > 256)
            return FP2_ERR_UNSUPPORTED;
        if (block % P->page_size != 0 && P->page_size % block != 0) return FP2_ERR_UNSUPPORTED;
        if (P->max_pages_per_seq < 1 || P->num_pages < 1) return FP2_ERR_INVALID_ARG;
    } else {
        if (P->total_k < 0) return FP2_ERR_INVALID_ARG;
    }
    return FP2_OK;
}

fp2_status check_dtype(const fp2_params* P, int block, fp2_dtype dtype) {
    if (P->out_dtype != FP2_BF16 && P->out_dtype != FP2_FP8_E4M3) return FP2_ERR_INVALID_ARG;
    if (P->out_dtype == FP2_FP8_E4M3 && dtype == FP2_BF16 && !P->out_scale)
        return FP2_ERR_INVALID_ARG;
    if (dtype == FP2_BF16) return (P->k_block_factor || P->v_block_factor) ? FP2_ERR_INVALID_ARG : FP2_OK;
    if (dtype != FP2_FP8_E4M3) return FP2_ERR_INVALID_ARG;
    if (P->head_dim != 128 || block != 128) return FP2_ERR_UNSUPPORTED;
    if (!P->q_scale || !P->k_scale || !P->v_scale) return FP2_ERR_INVALID_ARG;
    if (!P->k_block_factor != !P->v_block_factor) return FP2_ERR_INVALID_ARG;
    if (P->k_block_factor && P->attn_kernel != 0) return FP2_ERR_UNSUPPORTED;
    return FP2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void layout_of(const fp2_params* P, int block, fp2_workspace_layout* L) {
    const size_t S = (size_t)P->num_seqs, Hq = (size_t)P->num_q_heads,
                 Hkv = (size_t)P->num_kv_heads, d = (size_t)P->head_dim;
    // A call's query blocks follow the absolute blocks, so a sequence whose
    // prefix is not a multiple of the block spans up to one block more than
    // its queries alone would: ceil((P % B + Lq) / B) <= (Lq + 2B - 2) / B,
    // and never more than its keys' blocks.
    const int nkb = (P->max_seqlen_k + block - 1) / block;
    const int nqb = std::min((P->max_seqlen_q + 2 * block - 2) / block, nkb);
    const int nw = (nkb + 31) / 32;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    L->error_word = take(256);
    L->kbar = take(S * Hkv * nkb * d * 4);
    L->vbar = take(S * Hkv * nkb * d * 4);
    L->kbar_op = take(S * Hkv * nkb * d * 2);
    L->vbar_op = take(S * Hkv * nkb * d * 2);
    L->scores = take(S * Hq * nqb * nkb * 4);
    L->kept_idx = take(S * Hq * nqb * nkb * 4);
    L->kept_cnt = take(S * Hq * nqb * 4);
    L->kept_bits = take(S * Hq * nqb * nw * 4);
    L->total = o;
    L->nqb_max = nqb;
    L->nkb_max = nkb;
    L->nw = nw;
}

// Validates what every entry point needs and fills the kernel parameters.
// Entry points that take no dtype (mask, tau calibration) pass has_dtype =
// false: the input and output formats are then not theirs to check.
fp2_status prepare(const fp2_params* P, int block, fp2_dtype dtype, const int32_t* cu_seqlens,
                   const int32_t* page_table, KParams& kp, bool uses_kv = true,
                   bool has_dtype = true) {
    fp2_status st = check_params(P, block);
    if (st != FP2_OK) return st;
    if (has_dtype && (st = check_dtype(P, block, dtype)) != FP2_OK) return st;
    if ((st = check_kv(P, block, page_table)) != FP2_OK) return st;
    if (!cu_seqlens) return FP2_ERR_INVALID_ARG;
    fp2_workspace_layout L;
    layout_of(P, block, &L);
    if (!P->workspace || (reinterpret_cast<uintptr_t>(P->workspace) & 255u) != 0 ||
        P->workspace_bytes < L.total)
        return FP2_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(P->workspace);
    std::memset(&kp, 0, sizeof(kp));
    kp.num_seqs = P->num_seqs;
    kp.Hq = P->num_q_heads;
    kp.Hkv = P->num_kv_heads;
    kp.d = P->head_dim;
    kp.G = kp.Hq / kp.Hkv;
    kp.B = block;
    kp.total_q = P->total_q;
    kp.total_k = P->total_k;
    kp.paged = page_table ? 1 : 0;
    kp.page_size = page_table ? P->page_size : 0;
    kp.max_pages = page_table ? P->max_pages_per_seq : 0;
    kp.num_pages = page_table ? P->num_pages : 0;
    kp.max_seqlen_q = P->max_seqlen_q;
    kp.max_seqlen_k = P->max_seqlen_k;
    kp.nqb_max = L.nqb_max;
    kp.nkb_max = L.nkb_max;
    kp.nw = L.nw;
    kp.qb_lo = 0;
    kp.qb_n = L.nqb_max;
    kp.kb_lo = 0;
    kp.kb_n = L.nkb_max;
    kp.fp8 = dtype == FP2_FP8_E4M3;
    kp.uses_kv = uses_kv ? 1 : 0;
    kp.group_masks = P->group_masks ? 1 : 0;
    kp.out_fp8 = P->out_dtype == FP2_FP8_E4M3;
    kp.out_scale = P->out_scale;
    kp.attn_kernel = P->attn_kernel;
    kp.wait_limit_ns = (unsigned long long)P->debug_wait_limit_us * 1000ull;
    kp.withhold_k_item = P->debug_withhold_k_item;
    kp.kb_fac = P->k_block_factor;
    kp.vb_fac = P->v_block_factor;
    kp.cu_q = cu_seqlens;
    kp.cu_k = P->cu_seqlens_k ? P->cu_seqlens_k : cu_seqlens;
    kp.seqlens_k = P->seqlens_k;
    kp.page_table = page_table;
    kp.q_scale = P->q_scale;
    kp.k_scale = P->k_scale;
    kp.v_scale = P->v_scale;
    kp.err = reinterpret_cast<uint32_t*>(ws + L.error_word);
    kp.kbar = reinterpret_cast<float*>(ws + L.kbar);
    kp.vbar = reinterpret_cast<float*>(ws + L.vbar);
    kp.kbar_op = ws + L.kbar_op;
    kp.vbar_op = ws + L.vbar_op;
    kp.scores = reinterpret_cast<float*>(ws + L.scores);
    kp.kept_idx = reinterpret_cast<int32_t*>(ws + L.kept_idx);
    kp.kept_cnt = reinterpret_cast<int32_t*>(ws + L.kept_cnt);
    kp.kept_bits = reinterpret_cast<uint32_t*>(ws + L.kept_bits);
    return FP2_OK;
}

cudaStream_t stream_of(const fp2_params* P) { return static_cast<cudaStream_t>(P->stream); }

fp2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP2_OK : FP2_ERR_CUDA; }

// Events that order fp2_prefill_host's three streams: created once per device
// on first use, re-recorded by every call while g_host_mutex is held (so a
// record and the waits on it are never interleaved with another call's).
constexpr int kHostMaxChunks = 64;
constexpr int kHostEvents = 2 * kHostMaxChunks + 3;
constexpr int kHostMaxDevices = 64;
struct HostEvents {
    bool ready = false;
    cudaEvent_t ev[kHostEvents];
};
std::mutex g_host_mutex;
HostEvents g_host_events[kHostMaxDevices];

// `to` waits for the work queued so far on `from` (nothing when they are one stream)
cudaError_t join(cudaStream_t from, cudaStream_t to, cudaEvent_t e) {
    if (from == to) return cudaSuccess;
    cudaError_t r = cudaEventRecord(e, from);
    return r != cudaSuccess ? r : cudaStreamWaitEvent(to, e, 0);
}

}  // namespace

extern "C" {

const char* fp2_version(void) { return "0.1.0"; }

const char* fp2_status_string(fp2_status s) {
    switch (s) {
        case FP2_OK: return "ok";
        case FP2_ERR_INVALID_ARG: return "invalid argument";
        case FP2_ERR_UNSUPPORTED: return "unsupported configuration";
        case FP2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case FP2_ERR_CUDA: return "CUDA error";
        case FP2_ERR_TIMEOUT: return "device pipeline wait timed out";
        case FP2_ERR_DEVICE_BOUNDS: return "device index out of range";
    }
    return "unknown status";
}

size_t fp2_workspace_size(const fp2_params* params, int block) {
    if (check_params(params, block) != FP2_OK) return 0;
    fp2_workspace_layout L;
    layout_of(params, block, &L);
    return L.total;
}

fp2_status fp2_get_workspace_layout(const fp2_params* params, int block,
                                    fp2_workspace_layout* layout) {
    if (!layout) return FP2_ERR_INVALID_ARG;
    fp2_status st = check_params(params, block);
    if (st != FP2_OK) return st;
    layout_of(params, block, layout);
    return FP2_OK;
}

fp2_status fp2_blockmean(const void* k_cache, const void* v_cache, const int32_t* page_table,
                         const int32_t* cu_seqlens, int block, fp2_dtype dtype,
                         const fp2_params* params) {
    KParams kp;
    fp2_status st = prepare(params, block, dtype, cu_seqlens, page_table, kp);
    if (st != FP2_OK) return st;
    if (!k_cache || !v_cache) return FP2_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return FP2_ERR_INVALID_ARG;
    return cuda_status(fp2::launch_blockmean(kp, k_cache, v_cache, stream_of(params)));
}

static fp2_status attach_mean_cache(KParams& kp, const int32_t* block_table,
                                    int max_blocks_per_seq, float* mean_cache, int num_slots) {
    if (!block_table || !mean_cache || max_blocks_per_seq < 1 || num_slots < 1)
        return FP2_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mean_cache) & 15u) != 0) return FP2_ERR_INVALID_ARG;
    kp.mean_cache = mean_cache;
    kp.block_table = block_table;
    kp.max_blocks = max_blocks_per_seq;
    kp.num_slots = num_slots;
    return FP2_OK;
}

fp2_status fp2_blockmean_cached(const void* k_cache, const void* v_cache,
                                const int32_t* page_table, const int32_t* cu_seqlens,
                                const int32_t* block_table, int max_blocks_per_seq,
                                float* mean_cache, int num_slots, int block, fp2_dtype dtype,
                                const fp2_params* params) {
    KParams kp;
    fp2_status st = prepare(params, block, dtype, cu_seqlens, page_table, kp);
    if (st != FP2_OK) return st;
    if (!k_cache || !v_cache) return FP2_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return FP2_ERR_INVALID_ARG;
    if ((st = attach_mean_cache(kp, block_table, max_blocks_per_seq, mean_cache, num_slots)) !=
        FP2_OK)
        return st;
    return cuda_status(fp2::launch_blockmean(kp, k_cache, v_cache, stream_of(params)));
}

fp2_status fp2_score(const void* q, const int32_t* cu_seqlens, int block, fp2_dtype dtype,
                     const fp2_params* params) {
    KParams kp;
    fp2_status st = prepare(params, block, dtype, cu_seqlens, nullptr, kp, false);
    if (st != FP2_OK) return st;
    if (!q || !aligned16(q)) return FP2_ERR_INVALID_ARG;
    return cuda_status(fp2::launch_score(kp, q, stream_of(params)));
}

fp2_status fp2_mask(const int32_t* cu_seqlens, float tau, int block, const fp2_params* params) {
    KParams kp;
    fp2_status st = prepare(params, block, FP2_BF16, cu_seqlens, nullptr, kp, false, false);
    if (st != FP2_OK) return st;
    if (std::isnan(tau)) return FP2_ERR_INVALID_ARG;
    return cuda_status(fp2::launch_mask(kp, tau, stream_of(params)));
}

fp2_status fp2_attn(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* page_table, const int32_t* cu_seqlens,
                    const uint32_t* kept_bits, int block, fp2_dtype dtype, void* out,
                    const fp2_params* params) {
    KParams kp;
    fp2_status st = prepare(params, block, dtype, cu_seqlens, page_table, kp);
    if (st != FP2_OK) return st;
    if (!q || !k_cache || !v_cache || !out) return FP2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return FP2_ERR_INVALID_ARG;
    if (kp.total_q == 0) return FP2_OK;
    if (!page_table && kp.total_k == 0) return FP2_ERR_INVALID_ARG;
    const uint32_t* bits = kept_bits ? kept_bits : kp.kept_bits;
    cudaError_t e = fp2::launch_attn(kp, q, k_cache, v_cache, bits, out, stream_of(params));
    if (e == cudaErrorInvalidValue) return FP2_ERR_UNSUPPORTED;
    return cuda_status(e);
}

// Every check fp2_prefill makes before it queues anything; fills kp.
static fp2_status prefill_checks(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                                 int block, fp2_dtype dtype, const void* out,
                                 const fp2_params* params, const int32_t* block_table,
                                 int max_blocks_per_seq, float* mean_cache, int num_slots,
                                 KParams& kp) {
    fp2_status st = prepare(params, block, dtype, cu_seqlens, page_table, kp);
    if (st != FP2_OK) return st;
    if (mean_cache &&
        (st = attach_mean_cache(kp, block_table, max_blocks_per_seq, mean_cache, num_slots)) !=
            FP2_OK)
        return st;
    if (!q || !k_cache || !v_cache || !out) return FP2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return FP2_ERR_INVALID_ARG;
    if (std::isnan(tau)) return FP2_ERR_INVALID_ARG;
    if (kp.total_q > 0 && !page_table && kp.total_k == 0) return FP2_ERR_INVALID_ARG;
    return FP2_OK;
}

static fp2_status prefill_impl(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                               int block, fp2_dtype dtype, void* out, const fp2_params* params,
                               const int32_t* block_table, int max_blocks_per_seq,
                               float* mean_cache, int num_slots) {
    KParams kp;
    fp2_status st = prefill_checks(q, k_cache, v_cache, page_table, cu_seqlens, tau, block, dtype,
                                   out, params, block_table, max_blocks_per_seq, mean_cache,
                                   num_slots, kp);
    if (st != FP2_OK) return st;
    if (kp.total_q == 0) return FP2_OK;
    cudaStream_t s = stream_of(params);
    cudaError_t e = fp2::launch_blockmean(kp, k_cache, v_cache, s);
    kp.mean_cache = nullptr;  // only the block means use the cache
    if (e == cudaSuccess) e = fp2::launch_score(kp, q, s);
    if (e == cudaSuccess) e = fp2::launch_mask(kp, tau, s);
    if (e == cudaSuccess) e = fp2::launch_attn(kp, q, k_cache, v_cache, kp.kept_bits, out, s);
    if (e == cudaErrorInvalidValue) return FP2_ERR_UNSUPPORTED;
    return cuda_status(e);
}

fp2_status fp2_prefill(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                       int block, fp2_dtype dtype, void* out, const fp2_params* params) {
    return prefill_impl(q, k_cache, v_cache, page_table, cu_seqlens, tau, block, dtype, out,
                        params, nullptr, 0, nullptr, 0);
}

fp2_status fp2_prefill_cached(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                              int block, fp2_dtype dtype, void* out, const fp2_params* params,
                              const int32_t* block_table, int max_blocks_per_seq,
                              float* mean_cache, int num_slots) {
    if (!mean_cache) return FP2_ERR_INVALID_ARG;
    return prefill_impl(q, k_cache, v_cache, page_table, cu_seqlens, tau, block, dtype, out,
                        params, block_table, max_blocks_per_seq, mean_cache, num_slots);
}

fp2_status fp2_workspace_init(const fp2_params* params) {
    if (!params || !params->workspace || params->workspace_bytes < 256) return FP2_ERR_WORKSPACE;
    return cuda_status(cudaMemsetAsync(params->workspace, 0, 256, stream_of(params)));
}

fp2_status fp2_get_status(const fp2_params* params, uint32_t* detail) {
    if (!params || !params->workspace) return FP2_ERR_INVALID_ARG;
    cudaStream_t s = stream_of(params);
    uint32_t w[2] = {0, 0};
    if (cudaStreamSynchronize(s) != cudaSuccess) return FP2_ERR_CUDA;
    if (cudaMemcpy(w, params->workspace, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP2_ERR_CUDA;
    if (w[0] != 0) {
        if (cudaMemsetAsync(params->workspace, 0, sizeof(w), s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return FP2_ERR_CUDA;
    }
    if (detail) *detail = w[1];
    return static_cast<fp2_status>(w[0]);
}

fp2_status fp2_calibrate_tau(const int32_t* cu_seqlens, int block, float target_drop,
                             const fp2_params* params, float* tau_out) {
    KParams kp;
    fp2_status st = prepare(params, block, FP2_BF16, cu_seqlens, nullptr, kp, false, false);
    if (st != FP2_OK) return st;
    if (!tau_out || !(target_drop >= 0.f && target_drop <= 1.f)) return FP2_ERR_INVALID_ARG;
    cudaStream_t s = stream_of(params);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FP2_ERR_CUDA;
    const int S = kp.num_seqs;
    std::vector<int32_t> cu(S + 1), lk(S);
    if (cudaMemcpy(cu.data(), cu_seqlens, (S + 1) * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP2_ERR_CUDA;
    if (kp.seqlens_k) {
        if (cudaMemcpy(lk.data(), kp.seqlens_k, S * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
            return FP2_ERR_CUDA;
    } else {
        for (int b = 0; b < S; ++b) lk[b] = cu[b + 1] - cu[b];
    }
    std::vector<double> margins;
    size_t total = 0;
    std::vector<float> slab((size_t)kp.nqb_max * kp.nkb_max);
    for (int b = 0; b < S; ++b) {
        const int Lq = cu[b + 1] - cu[b];
        if (Lq < 0 || Lq > kp.max_seqlen_q || lk[b] < Lq || lk[b] > kp.max_seqlen_k)
            return FP2_ERR_INVALID_ARG;
        const int pb = (lk[b] - Lq) / block;
        const int nqb = Lq > 0 ? ((lk[b] - Lq) % block + Lq + block - 1) / block : 0;
        for (int h = 0; h < kp.Hq; ++h) {
            const size_t off = ((size_t)b * kp.Hq + h) * kp.nqb_max * kp.nkb_max;
            if (cudaMemcpy(slab.data(), kp.scores + off, (size_t)nqb * kp.nkb_max * 4,
                           cudaMemcpyDeviceToHost) != cudaSuccess)
                return FP2_ERR_CUDA;
            for (int i = 0; i < nqb; ++i) {
                const int iabs = pb + i;
                const float* row = slab.data() + (size_t)i * kp.nkb_max;
                total += (size_t)iabs + 1;
                double m = -INFINITY;
                for (int j = 0; j <= iabs; ++j) m = std::max(m, (double)row[j]);
                for (int j = 1; j < iabs; ++j) margins.push_back(m - (double)row[j]);
            }
        }
    }
    const size_t n = margins.size();
    if (n == 0) {
        *tau_out = INFINITY;
        return FP2_OK;
    }
    long long want = std::llround((double)target_drop * (double)total);
    want = std::max(0LL, std::min<long long>(want, (long long)n));
    if (want == 0) {
        *tau_out = (float)(*std::max_element(margins.begin(), margins.end()) + 1.0);
        return FP2_OK;
    }
    if (want == (long long)n) {
        const double lo = *std::min_element(margins.begin(), margins.end());
        *tau_out = (float)(lo > 0 ? lo / 2 : lo - 1.0);
        return FP2_OK;
    }
    const size_t k = n - (size_t)want;  // tau between the k-th and (k+1)-th smallest
    std::nth_element(margins.begin(), margins.begin() + k, margins.end());
    const double hi = margins[k];
    const double lo = *std::max_element(margins.begin(), margins.begin() + k);
    *tau_out = (float)(0.5 * (lo + hi));
    return FP2_OK;
}

fp2_status fp2_prefill_host(const fp2_host_io* io, const int32_t* page_table,
                            const int32_t* cu_seqlens, float tau, int block, fp2_dtype dtype,
                            const fp2_params* params) {
    if (!io || !params) return FP2_ERR_INVALID_ARG;
    if (io->num_chunks < 1 || io->num_chunks > kHostMaxChunks) return FP2_ERR_INVALID_ARG;
    if (!io->q_host || !io->k_host || !io->v_host || !io->out_host || !io->q_dev ||
        !io->k_dev || !io->v_dev || !io->out_dev || !io->cu_seqlens_host)
        return FP2_ERR_INVALID_ARG;
    if (params->seqlens_k && !io->seqlens_k_host) return FP2_ERR_INVALID_ARG;
    KParams kp;
    fp2_status st = prepare(params, block, dtype, cu_seqlens, page_table, kp);
    if (st != FP2_OK) return st;
    if (!aligned16(io->q_dev) || !aligned16(io->k_dev) || !aligned16(io->v_dev) ||
        !aligned16(io->out_dev))
        return FP2_ERR_INVALID_ARG;
    if (std::isnan(tau)) return FP2_ERR_INVALID_ARG;
    if (kp.total_q == 0) return FP2_OK;
    if (!page_table && kp.total_k == 0) return FP2_ERR_INVALID_ARG;

    // per-sequence geometry from the host copies of the lengths
    const int S = kp.num_seqs;
    const bool paged = page_table != nullptr;
    if (!paged && params->cu_seqlens_k && !io->cu_seqlens_k_host) return FP2_ERR_INVALID_ARG;
    const int32_t* cu = io->cu_seqlens_host;
    const int32_t* cuk = io->cu_seqlens_k_host ? io->cu_seqlens_k_host : cu;
    std::vector<int> q0(S), Lq(S), Lk(S), k0(S), off(S), pb(S);
    for (int b = 0; b < S; ++b) {
        q0[b] = cu[b];
        Lq[b] = cu[b + 1] - cu[b];
        Lk[b] = io->seqlens_k_host ? io->seqlens_k_host[b] : Lq[b];
        k0[b] = paged ? 0 : cuk[b];
        if (q0[b] < 0 || Lq[b] < 0 || Lq[b] > kp.max_seqlen_q || Lk[b] < Lq[b] ||
            Lk[b] > kp.max_seqlen_k || q0[b] + Lq[b] > kp.total_q ||
            (!paged && (k0[b] < 0 || k0[b] + Lk[b] > kp.total_k)))
            return FP2_ERR_INVALID_ARG;
        off[b] = (Lk[b] - Lq[b]) % block;
        pb[b] = (Lk[b] - Lq[b]) / block;
    }
    const size_t elt_in = kp.fp8 ? 1 : 2, elt_out = kp.out_fp8 ? 1 : 2;
    const size_t row_in = (size_t)kp.Hq * kp.d * elt_in, row_out = (size_t)kp.Hq * kp.d * elt_out;
    const size_t row_kv = (size_t)kp.Hkv * kp.d * elt_in;
    const size_t op_bytes = (size_t)S * kp.Hkv * kp.nkb_max * kp.d * elt_in;  // kbar_op / vbar_op

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP2_ERR_CUDA;
    if (dev < 0 || dev >= kHostMaxDevices) return FP2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_host_mutex);
    HostEvents& pool = g_host_events[dev];
    if (!pool.ready) {
        for (int e = 0; e < kHostEvents; ++e)
            if (cudaEventCreateWithFlags(&pool.ev[e], cudaEventDisableTiming) != cudaSuccess)
                return FP2_ERR_CUDA;
        pool.ready = true;
    }
    cudaEvent_t* ev = pool.ev;
    cudaStream_t s = stream_of(params);
    cudaStream_t up = io->upload_stream ? static_cast<cudaStream_t>(io->upload_stream) : s;
    cudaStream_t down = io->download_stream ? static_cast<cudaStream_t>(io->download_stream) : s;
    auto* qh = static_cast<const uint8_t*>(io->q_host);
    auto* qd = static_cast<uint8_t*>(io->q_dev);
    auto* kh = static_cast<const uint8_t*>(io->k_host);
    auto* kd = static_cast<uint8_t*>(io->k_dev);
    auto* vh = static_cast<const uint8_t*>(io->v_host);
    auto* vd = static_cast<uint8_t*>(io->v_dev);
    auto* oh = static_cast<uint8_t*>(io->out_host);
    auto* od = static_cast<const uint8_t*>(io->out_dev);
    auto h2d = [&](uint8_t* dst, const uint8_t* src, size_t at, size_t bytes) {
        return cudaMemcpyAsync(dst + at, src + at, bytes, cudaMemcpyHostToDevice, up);
    };

    // uploads start after the work already queued on params->stream
    cudaError_t e = join(s, up, ev[0]);
    int kb_done = 0;  // key blocks averaged so far
    if (paged) {
        // pages can sit anywhere in the cache: upload it whole, average every block
        const size_t kv_bytes = (size_t)kp.num_pages * kp.page_size * row_kv;
        if (e == cudaSuccess) e = h2d(kd, kh, 0, kv_bytes);
        if (e == cudaSuccess) e = h2d(vd, vh, 0, kv_bytes);
        if (e == cudaSuccess) e = join(up, s, ev[1]);
        if (e == cudaSuccess) e = fp2::launch_blockmean(kp, kd, vd, s);
        kb_done = kp.nkb_max;
    } else {
        // the mean tiles a range reads may reach blocks not averaged yet:
        // zeros there (weight-0 columns of PV must meet finite values)
        if (e == cudaSuccess) e = cudaMemsetAsync(kp.kbar_op, 0, op_bytes, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(kp.vbar_op, 0, op_bytes, s);
    }
    // query-block ranges, lowest first: a range needs the keys up to its last
    // diagonal block, so the key upload grows with the ranges.  Range c ends at
    // nqb * ((c+1)/n)^0.7: causal work grows with the query position, so the
    // early ranges are wider and the last ones, whose compute is the tail
    // after the uploads, narrower (measured: 0.7 beats even ranges by about
    // 1 % on the 128K layer; 0.6 does not)
    auto bound = [&](int c) {
        return (int)std::lround(kp.nqb_max * std::pow((double)c / io->num_chunks, 0.7));
    };
    for (int c = 0; e == cudaSuccess && c < io->num_chunks; ++c) {
        const int lo = bound(c), hi = std::min(kp.nqb_max, bound(c + 1));
        if (lo >= hi) continue;
        int kb_hi = kb_done;
        if (!paged) {
            for (int b = 0; b < S; ++b) kb_hi = std::max(kb_hi, pb[b] + hi);
            kb_hi = std::min(kb_hi, kp.nkb_max);
            for (int b = 0; e == cudaSuccess && b < S; ++b) {
                const int r0 = kb_done * block, r1 = std::min(Lk[b], kb_hi * block);
                if (r1 <= r0) continue;
                const size_t at = (size_t)(k0[b] + r0) * row_kv, bytes = (size_t)(r1 - r0) * row_kv;
                e = h2d(kd, kh, at, bytes);
                if (e == cudaSuccess) e = h2d(vd, vh, at, bytes);
            }
        }
        // the sequences' query rows of blocks [lo, hi): rows t with
        // lo <= (off + t) / B < hi
        for (int b = 0; e == cudaSuccess && b < S; ++b) {
            const int r0 = std::max(0, lo * block - off[b]);
            const int r1 = std::min(Lq[b], hi * block - off[b]);
            if (r1 > r0) e = h2d(qd, qh, (size_t)(q0[b] + r0) * row_in, (size_t)(r1 - r0) * row_in);
        }
        if (e == cudaSuccess) e = join(up, s, ev[2 + 2 * c]);
        if (e == cudaSuccess && kb_hi > kb_done) {
            kp.kb_lo = kb_done;
            kp.kb_n = kb_hi - kb_done;
            e = fp2::launch_blockmean(kp, kd, vd, s);
            kb_done = kb_hi;
        }
        kp.qb_lo = lo;
        kp.qb_n = hi - lo;
        if (e == cudaSuccess) e = fp2::launch_score(kp, qd, s);
        if (e == cudaSuccess) e = fp2::launch_mask(kp, tau, s);
        if (e == cudaSuccess) e = fp2::launch_attn(kp, qd, kd, vd, kp.kept_bits, io->out_dev, s);
        if (e == cudaSuccess) e = join(s, down, ev[3 + 2 * c]);
        for (int b = 0; e == cudaSuccess && b < S; ++b) {
            const int r0 = std::max(0, lo * block - off[b]);
            const int r1 = std::min(Lq[b], hi * block - off[b]);
            if (r1 > r0)
                e = cudaMemcpyAsync(oh + (size_t)(q0[b] + r0) * row_out, od + (size_t)(q0[b] + r0) * row_out,
                                    (size_t)(r1 - r0) * row_out, cudaMemcpyDeviceToHost, down);
        }
    }
    // blocks past every sequence's end get their zero means, as in fp2_prefill
    if (e == cudaSuccess && kb_done < kp.nkb_max) {
        kp.kb_lo = kb_done;
        kp.kb_n = kp.nkb_max - kb_done;
        e = fp2::launch_blockmean(kp, kd, vd, s);
    }
    // params->stream ends after the last download
    if (e == cudaSuccess) e = join(down, s, ev[kHostEvents - 1]);
    return cuda_status(e);
}

}  // extern "C"

namespace fp2 {
fp2_status validate_prefill(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                            int block, fp2_dtype dtype, const void* out,
                            const fp2_params* params) {
    KParams kp;
    return prefill_checks(q, k_cache, v_cache, page_table, cu_seqlens, tau, block, dtype, out,
                          params, nullptr, 0, nullptr, 0, kp);
}
}  // namespace fp2
