// fp2_stages.cu -- the three selection stages of FlashPrefill V2 on sm_100a:
//   blockmean: per-block means of K and V ("V_avg_dropped" of the popular
//              explainer, section 2.1) -- HBM-bound streaming reduction;
//   score:     pooled query blocks dotted with every causal key-block mean
//              (abstract: instantaneous pattern discovery) -- HBM-bound on Q;
//   mask:      max-based dynamic threshold with block 0 and the diagonal
//              always kept (abstract) -- one warp per (sequence, head, block).
// All three move 16-byte vectors and reduce with warp shuffles or a small
// shared-memory tree; none needs a tensor core.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp2_seq.cuh"

namespace fp2 {

template <bool FP8>
__device__ __forceinline__ void unpack16(const uint4& v, float* out) {
    if constexpr (FP8) {
        const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
            __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(b[e] | (b[e + 1] << 8));
            __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
            out[e] = f.x;
            out[e + 1] = f.y;
        }
    } else {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(h[e]);
            out[2 * e] = f.x;
            out[2 * e + 1] = f.y;
        }
    }
}

// ------------------------------------------------------------- blockmean ---
// grid (kb_n, num_seqs, ceil(Hkv*d / 1024)), 256 threads, one CTA per key
// block of one sequence and slice of at most 1024 of the Hkv*d columns (all
// KV heads when Hkv*d <= 1024).  The block's rows are contiguous in the cache
// (within a page, for a paged one), so they stream through shared memory by
// untiled bulk copies -- R rows of K and R of V per stage, kBmStages stages in
// flight -- while the threads add up the stage before: thread t owns columns
// 4t..4t+3 of the slice.  Blocks past the end of the sequence are written as
// zeros (the attention kernel reads whole tiles of means and multiplies the
// unused ones by zero).
constexpr int kBmThreads = 256, kBmStages = 3, kBmSlice = 4 * kBmThreads;
constexpr uint64_t kBmWaitNs = 2000000000ull;  // 2 s per stage wait

// rows per stage: at most 16 (they then never cross a page of >= 16 tokens)
// and at most 16 KB of one tensor
__host__ __device__ constexpr int bm_rows(int slice_bytes) {
    return slice_bytes <= 1024 ? 16 : (slice_bytes <= 2048 ? 8 : 4);
}

template <bool FP8>
__device__ __forceinline__ void unpack4(const uint8_t* src, float* out) {
    if constexpr (FP8) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w >> (8 * e)) & 0xFFFFu);
            __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
            out[e] = f.x;
            out[e + 1] = f.y;
        }
    } else {
        const uint2 w = *reinterpret_cast<const uint2*>(src);
        out[0] = __uint_as_float(w.x << 16);
        out[1] = __uint_as_float(w.x & 0xFFFF0000u);
        out[2] = __uint_as_float(w.y << 16);
        out[3] = __uint_as_float(w.y & 0xFFFF0000u);
    }
}

template <int D, bool FP8>
__global__ void __launch_bounds__(kBmThreads) blockmean_kernel(KParams p, const uint8_t* __restrict__ K,
                                                               const uint8_t* __restrict__ V) {
    constexpr int ELT = FP8 ? 1 : 2;
    extern __shared__ __align__(128) uint8_t bm_smem[];
    const int j = p.kb_lo + (int)blockIdx.x, b = blockIdx.y;
    const int W = p.Hkv * D;                               // columns of a row
    const int c0 = (int)blockIdx.z * kBmSlice;             // this CTA's columns
    const int WS = min(kBmSlice, W - c0);
    const size_t row_bytes = (size_t)W * ELT;
    const int R = bm_rows(WS * ELT);
    const int g = threadIdx.x, col = c0 + 4 * g;           // first of this thread's 4 columns
    const bool has_col = 4 * g < WS;

    SeqInfo s;
    if (!load_seq(p, b, s)) return;
    const int nkb = (s.Lk + p.B - 1) / p.B;
    auto out_at = [&](int c) {  // [S][Hkv][nkb_max][d] index of column c of block j
        return (((size_t)b * p.Hkv + c / D) * p.nkb_max + j) * D + (c % D);
    };
    if (j >= nkb) {
        if (has_col)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const size_t o = out_at(col + e);
                p.kbar[o] = 0.f;
                p.vbar[o] = 0.f;
                if constexpr (FP8) {
                    reinterpret_cast<uint8_t*>(p.kbar_op)[o] = 0;
                    reinterpret_cast<uint8_t*>(p.vbar_op)[o] = 0;
                } else {
                    reinterpret_cast<__nv_bfloat16*>(p.kbar_op)[o] = __float2bfloat16(0.f);
                    reinterpret_cast<__nv_bfloat16*>(p.vbar_op)[o] = __float2bfloat16(0.f);
                }
            }
        return;
    }
    const int t0 = j * p.B;
    const int n = min(p.B, s.Lk - t0);
    // block-mean cache: blocks wholly inside the resident prefix are read
    // from it, the others are computed and written back
    float* slot_ptr = nullptr;
    if (p.mean_cache) {
        const int slot = j < p.max_blocks ? p.block_table[(size_t)b * p.max_blocks + j] : -1;
        if (slot < 0 || slot >= p.num_slots) {
            set_error(p.err, kErrBounds, kDetSlot);
            return;
        }
        slot_ptr = p.mean_cache + (size_t)slot * 2 * W;
    }
    // per-block scale factors (e4m3 caches quantised per key block): the
    // means are dequantised with the block's scale and handed to the MMA in
    // units of the per-head scale, the unit of every mean tile
    auto emit = [&](int c, float mk, float mv) {  // mk, mv: means of the stored values
        const int hk = c / D;
        float fk = 1.f, fv = 1.f;
        if constexpr (FP8) {
            if (p.kb_fac) {
                const size_t fi = ((size_t)b * p.nkb_max + j) * p.Hkv + hk;
                fk = p.kb_fac[fi];
                fv = p.vb_fac[fi];
                if (!(fk > 0.f && fk <= 1.f && fv > 0.f && fv <= 1.f)) {
                    set_error(p.err, kErrInvalid, kDetFactor);
                    fk = fv = 1.f;
                }
            }
        }
        const size_t o = out_at(c);
        p.kbar[o] = mk * (FP8 ? p.k_scale[hk] * fk : 1.f);  // dequantised
        p.vbar[o] = mv * (FP8 ? p.v_scale[hk] * fv : 1.f);
        if constexpr (FP8) {
            reinterpret_cast<__nv_fp8_e4m3*>(p.kbar_op)[o] = __nv_fp8_e4m3(mk * fk);
            reinterpret_cast<__nv_fp8_e4m3*>(p.vbar_op)[o] = __nv_fp8_e4m3(mv * fv);
        } else {
            reinterpret_cast<__nv_bfloat16*>(p.kbar_op)[o] = __float2bfloat16(mk);
            reinterpret_cast<__nv_bfloat16*>(p.vbar_op)[o] = __float2bfloat16(mv);
        }
    };
    if (slot_ptr && t0 + p.B <= s.P) {
        if (has_col)
#pragma unroll
            for (int e = 0; e < 4; ++e) emit(col + e, slot_ptr[col + e], slot_ptr[W + col + e]);
        return;
    }

    // the ring: kBmStages barriers, then per stage R rows of K and R of V
    uint64_t* bars = reinterpret_cast<uint64_t*>(bm_smem);
    int* stage_rows = reinterpret_cast<int*>(bm_smem + 64);   // rows the stage holds
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bm_smem + 96);
    uint8_t* ring = bm_smem + 128;
    const size_t tile = (size_t)R * WS * ELT;                 // one tensor's rows of a stage
    const bool whole_rows = WS == W;                          // one copy per tensor and stage
    const int nst = (n + R - 1) / R;
    if (threadIdx.x == 0) {
        for (int k = 0; k < kBmStages; ++k) mbar_init(&bars[k], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // thread 0: stage st into slot st % kBmStages (rows of one page, or of the
    // contiguous cache)
    auto issue = [&](int st) {
        const int slot = st % kBmStages, r0 = st * R, nr = min(R, n - r0);
        const long long row = key_row(p, s, b, t0 + r0);
        uint64_t* bar = &bars[slot];
        stage_rows[slot] = row >= 0 ? nr : 0;
        const uint32_t dst = smem_u32(ring + slot * 2 * tile);
        if (row < 0) {
            mbar_arrive(bar);
        } else if (whole_rows) {
            const uint32_t bytes = (uint32_t)(nr * row_bytes);
            mbar_arrive_expect_tx(bar, 2 * bytes);
            bulk_load(dst, K + row * row_bytes, bytes, bar);
            bulk_load(dst + tile, V + row * row_bytes, bytes, bar);
        } else {
            const uint32_t bytes = (uint32_t)(WS * ELT);
            mbar_arrive_expect_tx(bar, 2 * bytes * nr);
            for (int r = 0; r < nr; ++r) {
                const size_t src = (row + r) * row_bytes + (size_t)c0 * ELT;
                bulk_load(dst + r * bytes, K + src, bytes, bar);
                bulk_load(dst + tile + r * bytes, V + src, bytes, bar);
            }
        }
    };
    if (threadIdx.x == 0)
        for (int st = 0; st < min(kBmStages - 1, nst); ++st) issue(st);
    float ak[4] = {0.f, 0.f, 0.f, 0.f}, av[4] = {0.f, 0.f, 0.f, 0.f};
    int issued = min(kBmStages - 1, nst), done = 0;
    for (int st = 0; st < nst; ++st) {
        if (threadIdx.x == 0 && issued < nst) issue(issued++);
        const bool ok = mbar_wait(&bars[st % kBmStages], (st / kBmStages) & 1, abort_flag, kBmWaitNs);
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) set_error(p.err, kErrTimeout, kDetWaitBase + 13);
            break;
        }
        const int slot = st % kBmStages, nr = stage_rows[slot];
        if (has_col) {
            const uint8_t* kt = ring + slot * 2 * tile + (size_t)4 * g * ELT;
            for (int r = 0; r < nr; ++r) {
                float fk[4], fv[4];
                unpack4<FP8>(kt + (size_t)r * WS * ELT, fk);
                unpack4<FP8>(kt + tile + (size_t)r * WS * ELT, fv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ak[e] += fk[e];
                    av[e] += fv[e];
                }
            }
        }
        done = st + 1;
        __syncthreads();  // the slot may be refilled
    }
    if (done < nst) {
        // aborted: let the copies already issued land before the CTA ends
        if (threadIdx.x == 0) {
            volatile int no_abort = 0;
            for (int st = done; st < issued; ++st)
                mbar_wait(&bars[st % kBmStages], (st / kBmStages) & 1, &no_abort, kBmWaitNs);
        }
        __syncthreads();
        return;
    }
    if (has_col) {
        const float inv = 1.f / (float)n;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float mk = ak[e] * inv, mv = av[e] * inv;
            emit(col + e, mk, mv);
            if (slot_ptr) {
                slot_ptr[col + e] = mk;
                slot_ptr[W + col + e] = mv;
            }
        }
    }
}

// ----------------------------------------------------------------- score ---
// grid (nqb_max, Hkv, num_seqs), 256 threads.  Pools the valid rows of one
// query block for the G query heads of one KV head (their rows are
// contiguous in q), then each warp takes 4 key blocks j <= i_abs at a time
// and forms their G dot products with kbar_j (lanes across d, reduce-scatter
// over the warp).
template <int D, bool FP8, int G>
__global__ void __launch_bounds__(256) score_kernel(KParams p, const uint8_t* __restrict__ Q) {
    constexpr int ELT = FP8 ? 1 : 2;
    constexpr int VEC = 16 / ELT;
    constexpr int VPT = G * D / VEC;          // 16-byte vectors per token (G heads)
    constexpr int TPP = 256 / VPT;            // tokens per pass
    static_assert(VPT <= 256 && 256 % VPT == 0, "tile shape");
    __shared__ float red[TPP][G * D];
    __shared__ float qb[G * D];

    const int i = p.qb_lo + (int)blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    SeqInfo s;
    if (!load_seq(p, b, s)) return;
    if (i >= s.nqb) return;
    // rows of query block i (the first may start inside its block)
    const int t0 = max(0, i * p.B - s.off);
    const int n = min(s.Lq, (i + 1) * p.B - s.off) - t0;
    const int iabs = s.pb + i;

    const int v = threadIdx.x % VPT, tg = threadIdx.x / VPT;
    float2 acc[VEC / 2];  // packed adds: half the issue slots
#pragma unroll
    for (int e = 0; e < VEC / 2; ++e) acc[e] = make_float2(0.f, 0.f);
    const uint8_t* qrow = Q + (((size_t)(s.q0 + t0) * p.Hq + hk * G) * D) * ELT + (size_t)v * 16;
    const size_t tok_stride = (size_t)p.Hq * D * ELT;
    // 8 loads in flight per thread before any is consumed
    constexpr int U = 8;
    int t = tg;
    for (; t + (U - 1) * TPP < n; t += U * TPP) {
        uint4 xs[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            xs[u] = __ldg(reinterpret_cast<const uint4*>(qrow + (size_t)(t + u * TPP) * tok_stride));
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float f[VEC];
            unpack16<FP8>(xs[u], f);
#pragma unroll
            for (int e = 0; e < VEC / 2; ++e) acc[e] = fadd2(acc[e], make_float2(f[2 * e], f[2 * e + 1]));
        }
    }
    for (; t < n; t += TPP) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(qrow + (size_t)t * tok_stride));
        float f[VEC];
        unpack16<FP8>(x, f);
#pragma unroll
        for (int e = 0; e < VEC / 2; ++e) acc[e] = fadd2(acc[e], make_float2(f[2 * e], f[2 * e + 1]));
    }
#pragma unroll
    for (int e = 0; e < VEC / 2; ++e) {
        red[tg][v * VEC + 2 * e] = acc[e].x;
        red[tg][v * VEC + 2 * e + 1] = acc[e].y;
    }
    __syncthreads();
    const float inv = 1.f / (float)n;
    for (int c = threadIdx.x; c < G * D; c += 256) {
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < TPP; ++r) sum += red[r][c];
        qb[c] = sum * inv * (FP8 ? p.q_scale[hk * G + c / D] : 1.f);
    }
    __syncthreads();
    if (p.group_masks && G > 1) {
        // group-shared masks: every head of the group is scored with the
        // mean of the G pooled queries (so all G get the same mask)
        float gm[(D + 255) / 256];
#pragma unroll
        for (int u = 0; u < (D + 255) / 256; ++u) {
            const int c = threadIdx.x + u * 256;
            float a = 0.f;
            if (c < D)
#pragma unroll
                for (int g = 0; g < G; ++g) a += qb[g * D + c];
            gm[u] = a / (float)G;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < (D + 255) / 256; ++u) {
            const int c = threadIdx.x + u * 256;
            if (c < D)
#pragma unroll
                for (int g = 0; g < G; ++g) qb[g * D + c] = gm[u];
        }
        __syncthreads();
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PER_LANE = D / 32;  // 4 (d=128) or 2 (d=64)
    constexpr int NV = 4 * G;         // 4 key blocks x G heads per warp step: 4 .. 32 values
    // Each warp takes 4 key blocks at a time: NV partial dot products per
    // lane (lanes split d), summed over the warp by a reduce-scatter
    // butterfly: the step with lane offset o (16, 8, ... while values remain)
    // halves what a lane carries, lanes with bit o set keeping the upper half
    // of the value indices.  So a lane ends up owning index m (below), and
    // its value slot x holds the product for index x ^ m: then the half a
    // lane keeps is always slots [0, half) and the half it sends [half, nv),
    // and the partner's sent slot x + half is the same index as the kept
    // slot x -- a shuffle and an add per value, no per-lane selects.
    int m = 0;
    {
        int h = NV >> 1;
#pragma unroll
        for (int o = 16; o >= 1 && h >= 1; o >>= 1, h >>= 1)
            if (lane & o) m += h;
    }
    const int m_r = m / G, m_g = m % G;  // index = key * G + head
    // pooled queries in this lane's head order (slot g holds head g ^ m_g)
    float2 qp[G][PER_LANE / 2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < PER_LANE / 2; ++e) {
            const float* src = qb + (g ^ m_g) * D + lane * PER_LANE + 2 * e;
            qp[g][e] = make_float2(src[0], src[1]);
        }
    const float scale = rsqrtf((float)D);
    const float* kb = p.kbar + ((size_t)b * p.Hkv + hk) * p.nkb_max * D + lane * PER_LANE;
    float* srow = p.scores + (((size_t)b * p.Hq + hk * G) * p.nqb_max + i) * p.nkb_max;
    const size_t head_stride = (size_t)p.nqb_max * p.nkb_max;
    for (int j0 = warp * 4; j0 <= iabs; j0 += 32) {
        float w[NV];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // slot r*G + g: key block j0 + (r ^ m_r), head g ^ m_g
            const int j = min(j0 + (r ^ m_r), iabs);
            float2 kv[PER_LANE / 2];
            if constexpr (PER_LANE == 4) {
                const float4 t4 = __ldg(reinterpret_cast<const float4*>(kb + (size_t)j * D));
                kv[0] = make_float2(t4.x, t4.y);
                kv[1] = make_float2(t4.z, t4.w);
            } else {
                kv[0] = __ldg(reinterpret_cast<const float2*>(kb + (size_t)j * D));
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float2 a = ffma2(qp[g][0], kv[0], make_float2(0.f, 0.f));
#pragma unroll
                for (int e = 1; e < PER_LANE / 2; ++e) a = ffma2(qp[g][e], kv[e], a);
                w[r * G + g] = a.x + a.y;
            }
        }
        int nv = NV;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            if (nv > 1) {
                const int half = nv >> 1;
#pragma unroll
                for (int x = 0; x < NV / 2; ++x)
                    if (x < half) w[x] += __shfl_xor_sync(0xffffffffu, w[x + half], o);
                nv = half;
            } else {
                w[0] += __shfl_xor_sync(0xffffffffu, w[0], o);
            }
        }
        constexpr int COPIES = 32 / NV;  // lanes holding the same value
        if ((lane & (COPIES - 1)) == 0) {
            const int j = j0 + m_r;
            if (j <= iabs) srow[(size_t)m_g * head_stride + j] = w[0] * scale;
        }
    }
}

// ------------------------------------------------------------------ mask ---
// One warp per (sequence, query head, query block): row maximum over the
// causal blocks, then keep j iff s_ij >= max - tau, or j == 0, or j == i_abs.
// Emits the kept bitmask (all nw words), the ascending kept list and count.
__global__ void __launch_bounds__(128) mask_kernel(KParams p, float tau) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // rows of this launch: (sequence, head) x query blocks [qb_lo, qb_lo + qb_n)
    const long long r = (long long)blockIdx.x * 4 + warp;
    if (r >= (long long)p.num_seqs * p.Hq * p.qb_n) return;
    const int i = p.qb_lo + (int)(r % p.qb_n);
    const long long bh = r / p.qb_n;  // b * Hq + h
    const int b = (int)(bh / p.Hq);
    const long long row = bh * p.nqb_max + i;  // [S][Hq][nqb_max] index
    SeqInfo s;
    if (!load_seq(p, b, s)) return;
    if (i >= s.nqb) return;
    const int iabs = s.pb + i;
    const float* S = p.scores + (size_t)row * p.nkb_max;
    float m = -INFINITY;
    for (int j = lane; j <= iabs; j += 32) m = fmaxf(m, S[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float thr = m - tau;
    int cnt = 0;
    uint32_t* bits = p.kept_bits + (size_t)row * p.nw;
    int32_t* idx = p.kept_idx + (size_t)row * p.nkb_max;
    const uint32_t below = (1u << lane) - 1u;
    for (int w = 0; w < p.nw; ++w) {
        const int j = w * 32 + lane;
        bool keep = false;
        if (j <= iabs) keep = (S[j] >= thr) || j == 0 || j == iabs;
        const uint32_t ball = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) bits[w] = ball;
        if (keep) idx[cnt + __popc(ball & below)] = j;
        cnt += __popc(ball);
    }
    if (lane == 0) p.kept_cnt[row] = cnt;
}

// -------------------------------------------------------------- launchers ---
cudaError_t launch_blockmean(const KParams& p, const void* k, const void* v, cudaStream_t st) {
    if (p.kb_n <= 0) return cudaSuccess;
    const int W = p.Hkv * p.d;
    if (W % 4 != 0) return cudaErrorInvalidValue;
    const int elt = p.fp8 ? 1 : 2;
    const int WS = W < kBmSlice ? W : kBmSlice;
    const size_t smem = 128 + (size_t)kBmStages * 2 * bm_rows(WS * elt) * WS * elt;
    dim3 grid(p.kb_n, p.num_seqs, (W + kBmSlice - 1) / kBmSlice);
    auto K = static_cast<const uint8_t*>(k);
    auto V = static_cast<const uint8_t*>(v);
    cudaError_t e = cudaSuccess;
    auto go = [&](auto kern) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) kern<<<grid, kBmThreads, smem, st>>>(p, K, V);
    };
    if (p.fp8) {
        if (p.d == 128) go(blockmean_kernel<128, true>);
        else go(blockmean_kernel<64, true>);
    } else {
        if (p.d == 128) go(blockmean_kernel<128, false>);
        else go(blockmean_kernel<64, false>);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, bool FP8>
static void score_dispatch_g(const KParams& p, const uint8_t* Q, dim3 grid, cudaStream_t st) {
    switch (p.G) {
        case 1: score_kernel<D, FP8, 1><<<grid, 256, 0, st>>>(p, Q); break;
        case 2: score_kernel<D, FP8, 2><<<grid, 256, 0, st>>>(p, Q); break;
        case 4: score_kernel<D, FP8, 4><<<grid, 256, 0, st>>>(p, Q); break;
        default: score_kernel<D, FP8, 8><<<grid, 256, 0, st>>>(p, Q); break;
    }
}

cudaError_t launch_score(const KParams& p, const void* q, cudaStream_t st) {
    dim3 grid(p.qb_n, p.Hkv, p.num_seqs);
    if (p.qb_n <= 0) return cudaSuccess;
    auto Q = static_cast<const uint8_t*>(q);
    if (p.fp8) {
        if (p.d == 128) score_dispatch_g<128, true>(p, Q, grid, st);
        else score_dispatch_g<64, true>(p, Q, grid, st);
    } else {
        if (p.d == 128) score_dispatch_g<128, false>(p, Q, grid, st);
        else score_dispatch_g<64, false>(p, Q, grid, st);
    }
    return cudaGetLastError();
}

cudaError_t launch_mask(const KParams& p, float tau, cudaStream_t st) {
    const long long rows = (long long)p.num_seqs * p.Hq * p.qb_n;
    if (rows <= 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + 3) / 4);
    mask_kernel<<<blocks, 128, 0, st>>>(p, tau);
    return cudaGetLastError();
}

}  // namespace fp2
