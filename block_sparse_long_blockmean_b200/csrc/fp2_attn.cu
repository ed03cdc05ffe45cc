// fp2_attn.cu -- block-sparse causal prefill attention with the block-mean
// correction on sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// What it computes (FlashPrefill V2 abstract: sparse attention operator,
// PackGQA memory access, warp specialisation, pipelining, mean correction
// term; popular explainer section 2.1): for every query row r of head h,
// an online softmax over
//   * the tokens of every key block h keeps (causal inside the diagonal
//     block), logit q.k/sqrt(d), value v;
//   * one pseudo-token per dropped causal block j (j < i_abs, not kept):
//     logit q.kbar_j/sqrt(d) + ln(n_j) with n_j = B (dropped blocks are
//     always full), value vbar_j.
//
// This one-tile kernel runs only when the caller asks for it
// (fp2_params.attn_kernel = 1; the two-tile kernel of fp2_attn_pair.cu takes
// every problem otherwise); the tests keep it as an independent second
// implementation of the same operator.
//
// Work item = (sequence, KV head, query block i, slice tq): 128 tensor-core
// rows = 128/G query tokens x the G query heads of the KV head (PackGQA: the
// K/V tile of a block is loaded once and used by all G heads).  The item
// walks the union of the G heads' kept blocks; rows of heads that did not
// keep a block mask it out.  After the kept blocks come "virtual" tiles of
// B block means (kbar, vbar) carrying the correction.
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then K/V (or mean) tiles into a
//               2-stage ring (paged K/V: one box per page)
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma:
//               S[n%2] = Q K_n^T  (SS, K-major),  O += P_{n-1} V_{n-1} (SS,
//               V MN-major)
//   warps 2..5  softmax warpgroup: thread = row = TMEM lane; reads S from
//               TMEM, masks, exponentiates (lazy rescale: O is rescaled
//               only when the running max grows by more than 2^8), writes P
//               (bf16 | e4m3) to shared memory in the 128-byte swizzle
//               layout, and at the end normalises O and stores bf16 rows.
// TMEM: S0 cols [0,128), S1 [128,256), O [256,256+d).
#include "fp2_attn_common.cuh"

namespace fp2 {

template <int D, int BLK, bool FP8>
struct AttnCfg {
    static constexpr int ELT = FP8 ? 1 : 2;
    static constexpr int CH = 128 / ELT;   // elements per 128-byte swizzle row
    static constexpr int NCH = D / CH;     // 128-byte chunks along d
    static constexpr int PCH = BLK / CH;   // 128-byte chunks along keys (P)
    static constexpr int M = 128;
    static constexpr int KSTEP = FP8 ? 32 : 16;
    static constexpr int Q_BYTES = M * D * ELT;
    static constexpr int KV_BYTES = BLK * D * ELT;
    static constexpr int P_BYTES = M * BLK * ELT;
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + 256;
    static constexpr int OFF_RING = OFF_MISC + 64;  // page ids of upcoming items
    static constexpr int OFF_ITEMS = OFF_RING + kPageRing * kMaxBoxes * 4;
    static_assert(NCH >= 1 && PCH >= 1, "tile shape");
    static_assert(D % 32 == 0 && BLK % 32 == 0, "tile shape");
};

// barrier slots
enum { B_KV_FULL = 0, B_KV_EMPTY = 2, B_S_FULL = 4, B_S_FREE = 6, B_Q_FULL = 8, B_P_READY = 9,
       B_O_DONE = 10, B_DRAIN = 11, B_COUNT = 12 };

template <int D, int BLK, bool FP8>
__global__ void __launch_bounds__(192, 1)
attn_kernel(const KParams p, const __grid_constant__ AttnMaps maps,
            const uint32_t* __restrict__ kept_bits, __nv_bfloat16* __restrict__ out,
            int items_cap) {
    using C = AttnCfg<D, BLK, FP8>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the swizzled tiles (shared address space)
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    int* items = reinterpret_cast<int*>(smem + C::OFF_ITEMS);
    uint32_t* sbits = reinterpret_cast<uint32_t*>(items + items_cap);  // [G][nw_c]

    const int G = p.G;
    const int TOK = 128 / G;
    const int ntq = BLK / TOK;
    // longest-first order: the largest query block index goes first
    const int per_i = p.num_seqs * p.Hkv * ntq;
    const int i = p.qb_lo + p.qb_n - 1 - (int)(blockIdx.x / per_i);
    const int rem = (int)(blockIdx.x % per_i);
    const int b = rem / (p.Hkv * ntq);
    const int hk = (rem / ntq) % p.Hkv;
    const int tq = rem % ntq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;

    SeqInfo s;
    if (!load_seq(p, b, s)) return;
    // the tile's first query (negative inside a partial first query block)
    const int t_begin = i * BLK - s.off + tq * TOK;
    if (i >= s.nqb || t_begin >= s.Lq || t_begin + TOK <= 0) return;  // no rows here
    const int iabs = s.pb + i;
    const int nw_c = (iabs + 32) / 32;  // words covering blocks 0..iabs

    // ---------------------------------------------------------- set-up ---
    if (threadIdx.x == 0) {
        for (int k = 0; k < B_COUNT; ++k) {
            uint32_t cnt = 1;
            if (k == B_S_FREE || k == B_S_FREE + 1 || k == B_P_READY) cnt = 128;
            mbar_init(&bars[k], cnt);
        }
        misc[1] = 0;  // abort flag
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    load_kept_bits(p, kept_bits, b, hk, i, iabs, nw_c, sbits);
    __syncthreads();
    if (warp == 0) {
        const int n = build_items<BLK>(G, iabs, nw_c, sbits, items);
        if (lane == 0) misc[2] = (uint32_t)n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int n_items = (int)misc[2];

    const uint32_t q_s = sbase + C::OFF_Q;
    const uint32_t p_s = sbase + C::OFF_P;

    if (warp == 0) {
        // ------------------------------------------------------ producer ---
        // the whole warp resolves page ids 32 items at a time; lane 0 waits
        // and issues every copy
        int* pring = reinterpret_cast<int*>(smem + C::OFF_RING);
        if (lane == 0) {
            prefetch_tmap(&maps.q);
            prefetch_tmap(&maps.k);
            prefetch_tmap(&maps.v);
            mbar_arrive_expect_tx(&bars[B_Q_FULL], C::Q_BYTES);
            for (int c = 0; c < C::NCH; ++c)
                tma_load_3d(q_s + c * (128 * 128), &maps.q, &bars[B_Q_FULL], c * C::CH, hk * G,
                            s.q0 + t_begin);
        }
        int issued = 0;
        bool ok = true;
        for (int n = 0; n < n_items; ++n) {
            if (n % 32 == 0) fill_page_ring<BLK>(p, s, b, items, n_items, n, pring);
            if (lane == 0) {
                const int st = n & 1;
                if (n >= 2 && !mbar_wait(&bars[B_KV_EMPTY + st], ((n - 2) >> 1) & 1, abort_flag,
                                         wlim)) {
                    set_error(p.err, kErrTimeout, kDetWaitBase + 0);
                    ok = false;
                } else {
                    issue_item_loads<D, BLK, FP8>(p, maps, s, b, hk, items[n],
                                                  pring + (n % kPageRing) * kMaxBoxes,
                                                  sbase + C::OFF_K + st * C::KV_BYTES,
                                                  sbase + C::OFF_V + st * C::KV_BYTES,
                                                  &bars[B_KV_FULL + st]);
                    ++issued;
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
        if (lane == 0) {
            // never leave with copies in flight: wait (bounded) for the loads
            // of the last two stages, whatever happened above
            volatile int no_abort = 0;
            for (int n = max(0, issued - 2); n < issued; ++n)
                mbar_wait(&bars[B_KV_FULL + (n & 1)], (n >> 1) & 1, &no_abort, wlim);
            mbar_wait(&bars[B_Q_FULL], 0, &no_abort, wlim);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issue ---
        if (lane == 0) {
            constexpr uint32_t fmt = FP8 ? 0u : 1u;
            constexpr uint32_t idesc_qk = make_idesc(fmt, false, 128, BLK);
            constexpr uint32_t idesc_pv = make_idesc(fmt, true, 128, D);
            const uint32_t o_tmem = tmem + 256;
            bool ok = mbar_wait(&bars[B_Q_FULL], 0, abort_flag, wlim);
            if (!ok) set_error(p.err, kErrTimeout, kDetWaitBase + 1);
            tc_fence_after();
            for (int n = 0; ok && n <= n_items; ++n) {
                if (n < n_items) {
                    const int st = n & 1;
                    if (!mbar_wait(&bars[B_KV_FULL + st], (n >> 1) & 1, abort_flag, wlim) ||
                        (n >= 2 &&
                         !mbar_wait(&bars[B_S_FREE + st], ((n - 2) >> 1) & 1, abort_flag,
                                    wlim))) {
                        set_error(p.err, kErrTimeout, kDetWaitBase + 2);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_s = sbase + C::OFF_K + st * C::KV_BYTES;
                    const uint32_t s_tmem = tmem + st * 128;
#pragma unroll
                    for (int ks = 0; ks < D / C::KSTEP; ++ks) {
                        const int ch = (ks * C::KSTEP) / C::CH;
                        const uint32_t within = (uint32_t)((ks * C::KSTEP) % C::CH) * C::ELT;
                        const uint64_t ad = sw128_desc(q_s + ch * (128 * 128) + within, 16, 1024);
                        const uint64_t bd = sw128_desc(k_s + ch * (BLK * 128) + within, 16, 1024);
                        if constexpr (FP8) mma_f8_ss(s_tmem, ad, bd, idesc_qk, ks > 0);
                        else mma_bf16_ss(s_tmem, ad, bd, idesc_qk, ks > 0);
                    }
                    mma_commit(&bars[B_S_FULL + st]);
                }
                if (n >= 1) {
                    const int m = n - 1;
                    const int stp = m & 1;
                    if (!mbar_wait(&bars[B_P_READY], m & 1, abort_flag, wlim)) {
                        set_error(p.err, kErrTimeout, kDetWaitBase + 3);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t v_s = sbase + C::OFF_V + stp * C::KV_BYTES;
#pragma unroll
                    for (int ks = 0; ks < BLK / C::KSTEP; ++ks) {
                        const int ch = (ks * C::KSTEP) / C::CH;
                        const uint32_t within = (uint32_t)((ks * C::KSTEP) % C::CH) * C::ELT;
                        const uint64_t ad = sw128_desc(p_s + ch * (128 * 128) + within, 16, 1024);
                        const uint64_t bd = sw128_desc(v_s + ks * C::KSTEP * 128, BLK * 128, 1024);
                        const uint32_t acc = (m > 0 || ks > 0) ? 1u : 0u;
                        if constexpr (FP8) mma_f8_ss(o_tmem, ad, bd, idesc_pv, acc);
                        else mma_bf16_ss(o_tmem, ad, bd, idesc_pv, acc);
                    }
                    mma_commit(&bars[B_O_DONE]);
                    mma_commit(&bars[B_KV_EMPTY + stp]);
                }
            }
            // all MMAs of this thread complete before the CTA may release TMEM
            mma_commit(&bars[B_DRAIN]);
            volatile int no_abort = 0;
            mbar_wait(&bars[B_DRAIN], 0, &no_abort, wlim);
        }
    } else {
        // ------------------------------------------------ softmax warpgroup ---
        const int qw = warp & 3;                 // TMEM lane quarter of this warp
        const int r = qw * 32 + lane;            // tile row == TMEM lane
        const int g = r % G;
        const int tl = r / G;
        const int t = t_begin + tl;              // query index in the sequence
        const int h = hk * G + g;
        const bool row_ok = t >= 0 && t < s.Lq;
        const int ppos = s.P + t;                // absolute position
        const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
        const uint32_t o_addr = tmem + lane_off + 256;
        const uint32_t* hb = sbits + g * nw_c;
        float sl2 = rsqrtf((float)D) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
        if constexpr (FP8) sl2 *= p.q_scale[h] * p.k_scale[hk];
        const float lb = __log2f((float)BLK);    // log2(n_j), n_j = BLK for dropped blocks
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int n = 0; n < n_items; ++n) {
            const int st = n & 1;
            // the row's columns of this item, from shared memory, decided
            // before S is waited for so the loads' latency hides behind it
            const int item = items[n];
            int lim = -1;                // real tile: last column taken
            uint32_t dropped[BLK / 32];  // mean tile: the row's dropped blocks
            if (item >= 0) {
                const bool kept = row_ok && ((hb[item >> 5] >> (item & 31)) & 1u);
                lim = !kept ? -1 : (item == iabs ? ppos - item * BLK : BLK - 1);
            } else {
                const int tv = -item - 1;
#pragma unroll
                for (int w = 0; w < BLK / 32; ++w) {
                    const int j0 = tv * BLK + w * 32;  // multiple of 32
                    uint32_t dm = 0u;
                    if (row_ok && j0 < iabs) {
                        dm = ~hb[j0 >> 5];
                        const int nvalid = iabs - j0;
                        if (nvalid < 32) dm &= (1u << nvalid) - 1u;
                    }
                    dropped[w] = dm;
                }
            }
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&bars[B_S_FULL + st], (n >> 1) & 1, abort_flag, wlim))) {
                set_error(p.err, kErrTimeout, kDetWaitBase + 4);
                ok = false;
                break;
            }
            tc_fence_after();
            float x[BLK];
#pragma unroll
            for (int c = 0; c < BLK / 32; ++c)
                tmem_ld32f(tmem + lane_off + st * 128 + c * 32, x + c * 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[B_S_FREE + st]);

            float mx = -INFINITY;
            if (item >= 0) {
#pragma unroll
                for (int c = 0; c < BLK; ++c) {
                    const float v = c <= lim ? x[c] * sl2 : -INFINITY;
                    x[c] = v;
                    mx = fmaxf(mx, v);
                }
            } else {
#pragma unroll
                for (int w = 0; w < BLK / 32; ++w)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float v = ((dropped[w] >> e) & 1u) ? fmaf(x[w * 32 + e], sl2, lb)
                                                                : -INFINITY;
                        x[w * 32 + e] = v;
                        mx = fmaxf(mx, v);
                    }
            }
            float alpha = 1.f;
            bool rescale = false;
            if (m_used == -INFINITY) {
                m_used = mx;  // O row is still exactly zero: nothing to rescale
            } else if (mx > m_used + kRescaleLog2) {
                alpha = ex2(m_used - mx);
                m_used = mx;
                rescale = true;
            }
            const float mb = m_used == -INFINITY ? 0.f : m_used;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < BLK; ++c) {
                const float pv = ex2(x[c] - mb);
                x[c] = pv;
                sum += pv;
            }
            l = l * alpha + sum;

            // PV of the previous item must be complete before P and O change
            if (n >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[B_O_DONE], (n - 1) & 1,
                                                             abort_flag, wlim))) {
                set_error(p.err, kErrTimeout, kDetWaitBase + 5);
                ok = false;
                break;
            }
            tc_fence_after();
            // P row -> shared memory, 128-byte swizzle, K-major (keys)
            uint8_t* prow = smem + C::OFF_P + r * 128;
#pragma unroll
            for (int pc = 0; pc < C::PCH; ++pc) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint4 w;
                    if constexpr (FP8) {
                        const float* src = x + pc * 128 + u * 16;
                        uint32_t wd[4];
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                                make_float2(src[4 * q4], src[4 * q4 + 1]), __NV_SATFINITE, __NV_E4M3);
                            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                                make_float2(src[4 * q4 + 2], src[4 * q4 + 3]), __NV_SATFINITE, __NV_E4M3);
                            wd[q4] = (uint32_t)lo | ((uint32_t)hi << 16);
                        }
                        w = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    } else {
                        const float* src = x + pc * 64 + u * 8;
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(src[0], src[1]);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(src[2], src[3]);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(src[4], src[5]);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(src[6], src[7]);
                        w = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                       *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                    }
                    *reinterpret_cast<uint4*>(prow + pc * (128 * 128) + ((u ^ (r & 7)) * 16)) = w;
                }
            }
            // a partial last key block: zero the V rows past the sequence end
            // (they may hold stale page contents; P is zero there, but 0 * NaN
            // would not be)
            if (item >= 0 && item * BLK + BLK > s.Lk)
                zero_v_tail<BLK, C::NCH>(smem + C::OFF_V + st * C::KV_BYTES,
                                         max(0, s.Lk - item * BLK), r, 128);
            if (__any_sync(0xffffffffu, rescale && n >= 1)) {
                const float a = (rescale && n >= 1) ? alpha : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + 256 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
                    tmem_st32(tmem + lane_off + 256 + c * 32, o);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_P_READY]);
        }
        // ------------------------------------------------------- epilogue ---
        if (ok && __all_sync(0xffffffffu, mbar_wait(&bars[B_O_DONE], (n_items - 1) & 1,
                                                    abort_flag, wlim))) {
            tc_fence_after();
            float inv = l > 0.f ? 1.f / l : 0.f;
            if (p.out_fp8) {
                // e4m3 output in units of out_scale[h] (default: the KV head's
                // v_scale, the units O has before dequantisation)
                float vs = FP8 ? p.v_scale[hk] : 1.f;
                if (p.out_scale) inv *= vs / p.out_scale[h];
                else if (!FP8) inv = 0.f;  // rejected on the host; never reached
                uint8_t* orow8 = reinterpret_cast<uint8_t*>(out) + ((size_t)(s.q0 + t) * p.Hq + h) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + c * 32, o);
                    tmem_wait_ld();
                    if (row_ok) {
                        uint32_t wd[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            wd[e] = pack_e4m3x4(__uint_as_float(o[4 * e]) * inv,
                                                __uint_as_float(o[4 * e + 1]) * inv,
                                                __uint_as_float(o[4 * e + 2]) * inv,
                                                __uint_as_float(o[4 * e + 3]) * inv);
                        *reinterpret_cast<uint4*>(orow8 + c * 32) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                        *reinterpret_cast<uint4*>(orow8 + c * 32 + 16) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
                    }
                }
            } else {
            if constexpr (FP8) inv *= p.v_scale[hk];
            __nv_bfloat16* orow = out + ((size_t)(s.q0 + t) * p.Hq + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(o_addr + c * 32, o);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint32_t wd[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 hh = __floats2bfloat162_rn(
                                __uint_as_float(o[u * 8 + 2 * e]) * inv,
                                __uint_as_float(o[u * 8 + 2 * e + 1]) * inv);
                            wd[e] = *reinterpret_cast<uint32_t*>(&hh);
                        }
                        *reinterpret_cast<uint4*>(orow + c * 32 + u * 8) =
                            make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    }
                }
            }
            }
        } else if (ok) {
            set_error(p.err, kErrTimeout, kDetWaitBase + 6);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------ host side ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

static bool encode(CUtensorMap* m, bool fp8, int rank, const void* base, const cuuint64_t* dims,
                   const cuuint64_t* strides, const cuuint32_t* box) {
    EncodeTiledFn fn = get_encode();
    if (!fn) return false;
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_attn_maps(const KParams& p, const void* q, const void* k, const void* v, int D,
                    int BLK, int TOK, AttnMaps* maps) {
    const bool fp8 = p.fp8 != 0;
    const cuuint64_t E = fp8 ? 1 : 2;
    const cuuint32_t CH = fp8 ? 128 : 64;
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.Hq, (cuuint64_t)p.total_q};
        cuuint64_t str[2] = {D * E, (cuuint64_t)p.Hq * D * E};
        cuuint32_t box[3] = {CH, (cuuint32_t)p.G, (cuuint32_t)TOK};
        if (!encode(&maps->q, fp8, 3, q, dims, str, box)) return false;
    }
    if (!p.paged) {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.Hkv, (cuuint64_t)p.total_k};
        cuuint64_t str[2] = {D * E, (cuuint64_t)p.Hkv * D * E};
        cuuint32_t box[3] = {CH, 1, (cuuint32_t)BLK};
        if (!encode(&maps->k, fp8, 3, k, dims, str, box)) return false;
        if (!encode(&maps->v, fp8, 3, v, dims, str, box)) return false;
    } else {
        const int R = p.page_size < BLK ? p.page_size : BLK;
        cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.Hkv, (cuuint64_t)p.page_size,
                              (cuuint64_t)p.num_pages};
        cuuint64_t str[3] = {D * E, (cuuint64_t)p.Hkv * D * E,
                             (cuuint64_t)p.page_size * p.Hkv * D * E};
        cuuint32_t box[4] = {CH, 1, (cuuint32_t)R, 1};
        if (!encode(&maps->k, fp8, 4, k, dims, str, box)) return false;
        if (!encode(&maps->v, fp8, 4, v, dims, str, box)) return false;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.nkb_max,
                              (cuuint64_t)p.num_seqs * p.Hkv};
        cuuint64_t str[2] = {D * E, (cuuint64_t)p.nkb_max * D * E};
        cuuint32_t box[3] = {CH, (cuuint32_t)BLK, 1};
        if (!encode(&maps->kb, fp8, 3, p.kbar_op, dims, str, box)) return false;
        if (!encode(&maps->vb, fp8, 3, p.vbar_op, dims, str, box)) return false;
    }
    return true;
}

template <int D, int BLK, bool FP8>
static cudaError_t launch_attn_t(const KParams& p, const void* q, const void* k, const void* v,
                                 const uint32_t* kept_bits, void* out, cudaStream_t st) {
    using C = AttnCfg<D, BLK, FP8>;
    AttnMaps maps;
    const int TOK = 128 / p.G;
    if (!make_attn_maps(p, q, k, v, D, BLK, TOK, &maps)) return cudaErrorInvalidValue;
    const int items_cap = p.nkb_max + (p.nkb_max + BLK - 1) / BLK + 2;
    const int nw_c_max = p.nkb_max / 32 + 1;
    size_t smem = 1024 + C::OFF_ITEMS + (size_t)items_cap * 4 + (size_t)p.G * nw_c_max * 4;
    const size_t min_smem = 120 * 1024;  // one CTA per SM (it owns all 512 TMEM columns)
    if (smem < min_smem) smem = min_smem;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, BLK, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int ntq = BLK / TOK;
    const long long grid = (long long)p.qb_n * p.num_seqs * p.Hkv * ntq;
    if (grid <= 0) return cudaSuccess;
    attn_kernel<D, BLK, FP8><<<(unsigned)grid, 192, smem, st>>>(
        p, maps, kept_bits, static_cast<__nv_bfloat16*>(out), items_cap);
    return cudaGetLastError();
}

cudaError_t launch_attn_pair(const KParams& p, const void* q, const void* k, const void* v,
                             const uint32_t* kept_bits, void* out, cudaStream_t st);

// Every problem goes to the two-tile kernel unless the caller selected the
// one-tile kernel above (KParams::attn_kernel = 1).
cudaError_t launch_attn(const KParams& p, const void* q, const void* k, const void* v,
                        const uint32_t* kept_bits, void* out, cudaStream_t st) {
    if (p.attn_kernel == 0) return launch_attn_pair(p, q, k, v, kept_bits, out, st);
    if (p.fp8) {
        if (p.d == 128 && p.B == 128) return launch_attn_t<128, 128, true>(p, q, k, v, kept_bits, out, st);
        return cudaErrorInvalidValue;
    }
    if (p.d == 128 && p.B == 128) return launch_attn_t<128, 128, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 128 && p.B == 64) return launch_attn_t<128, 64, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 64 && p.B == 128) return launch_attn_t<64, 128, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 64 && p.B == 64) return launch_attn_t<64, 64, false>(p, q, k, v, kept_bits, out, st);
    return cudaErrorInvalidValue;
}

}  // namespace fp2
