// fp2_attn_common.cuh -- pieces shared by the two attention kernels:
// tensor maps, the per-CTA work list (union of the G heads' kept blocks,
// then the block-mean tiles that carry the correction), and the TMA issue of
// one K/V (or mean) tile into a pipeline stage.  The work list is the
// PackGQA walk (FlashPrefill V2 popular explainer, section 2.2 kernel layer:
// the G query heads of a KV head share each K/V tile); the mean tiles carry
// the dropped blocks' constant term (same explainer, section 2.1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp2_seq.cuh"

namespace fp2 {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait
constexpr float kRescaleLog2 = 8.0f;              // lazy-rescale threshold (x256)

struct AttnMaps {
    CUtensorMap q, k, v, kb, vb;
};

// Host: encodes the five tensor maps of an attention launch (Q boxes of
// tok x G rows; K/V boxes of one key block or one page; mean-tile boxes).
bool make_attn_maps(const KParams& p, const void* q, const void* k, const void* v, int D,
                    int BLK, int TOK, AttnMaps* maps);

// Loads the G heads' kept bits of query block i into sbits[G][nw_c] (block 0
// and the diagonal forced on, bits past the diagonal cleared).  All threads.
__device__ __forceinline__ void load_kept_bits(const KParams& p, const uint32_t* kept_bits, int b,
                                               int hk, int i, int iabs, int nw_c, uint32_t* sbits) {
    const int G = p.G;
    const uint32_t* src = kept_bits + (((size_t)b * p.Hq + (size_t)hk * G) * p.nqb_max + i) * p.nw;
    for (int x = threadIdx.x; x < G * nw_c; x += blockDim.x) {
        const int g = x / nw_c, w = x % nw_c;
        uint32_t word = src[(size_t)g * p.nqb_max * p.nw + w];
        if (w == 0) word |= 1u;
        if (w == (iabs >> 5)) {
            word |= 1u << (iabs & 31);
            const int hi = iabs & 31;
            if (hi < 31) word &= (2u << hi) - 1u;
        }
        sbits[x] = word;
    }
}

// One warp: writes the work list into items[] and returns its length.
//   item >= 0 : key block j kept by at least one of the G heads (ascending)
//   item <  0 : -(t+1), the tile of block means [t*BLK, t*BLK+BLK) that holds
//               at least one block some head dropped (blocks < iabs)
template <int BLK>
__device__ __forceinline__ int build_items(int G, int iabs, int nw_c, const uint32_t* sbits,
                                           int* items) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int w0 = 0; w0 < nw_c; w0 += 32) {
        const int w = w0 + lane;
        uint32_t u = 0;
        if (w < nw_c)
            for (int g = 0; g < G; ++g) u |= sbits[g * nw_c + w];
        const int c = __popc(u);
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        int pos = base + incl - c;
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1;
            items[pos++] = w * 32 + bit;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int nvt = (iabs + BLK - 1) / BLK;
    for (int t = 0; t < nvt; ++t) {
        const int lo = t * BLK, hi = min(iabs, (t + 1) * BLK);  // blocks [lo, hi)
        const int w_lo = lo >> 5, nwt = ((hi + 31) >> 5) - w_lo;
        bool any = false;
        for (int x = lane; x < G * nwt; x += 32) {
            const int g = x / nwt, w = w_lo + x % nwt;
            uint32_t m = ~sbits[g * nw_c + w];
            const int top = hi - w * 32;  // > 0
            if (top < 32) m &= (1u << top) - 1u;
            any |= (m != 0u);
        }
        any = __any_sync(0xffffffffu, any);
        if (lane == 0 && any) items[base] = -(t + 1);
        if (any) ++base;
    }
    return base;
}

// Issues the TMA loads of ONE operand tile of a work item (the K tile, or
// the V tile: `map`/`mean_map` select which) into `dst` (NCH 128-byte chunks
// of BLK rows) and adds the bytes that will land to `full`'s current phase.
// `arrive`: also arrive on `full` (its arrival count is 1, so exactly one
// call per phase may arrive; others only add their bytes).  Paged keys
// load one box per page that holds keys of the block; pages past the
// sequence end are skipped (their rows are never used: the diagonal mask
// drops them and the V rows are zeroed).
template <int D, int BLK, bool FP8>
__device__ __forceinline__ void issue_tile_load(const KParams& p, const CUtensorMap* map,
                                                const CUtensorMap* mean_map, const SeqInfo& s,
                                                int b, int hk, int item, const int* pages,
                                                uint32_t dst, uint64_t* full, bool arrive) {
    constexpr int ELT = FP8 ? 1 : 2;
    constexpr int CH = 128 / ELT;
    constexpr int NCH = D / CH;
    constexpr int TILE_BYTES = BLK * D * ELT;
    if (item >= 0) {
        const int j = item;
        if (!p.paged) {
            if (arrive) mbar_arrive_expect_tx(full, TILE_BYTES);
            else mbar_expect_tx(full, TILE_BYTES);
#pragma unroll
            for (int c = 0; c < NCH; ++c)
                tma_load_3d(dst + c * BLK * 128, map, full, c * CH, hk, s.k0 + j * BLK);
        } else {
            // pages[sb]: physical page of rows [sb*R, sb*R+R) of the block, or
            // -1 (past the sequence end / invalid id: not loaded)
            const int R = min(p.page_size, BLK);
            int nbox = 0;
            for (int sb = 0; sb < BLK / R; ++sb) nbox += (pages[sb] >= 0);
            if (arrive) mbar_arrive_expect_tx(full, (uint32_t)(nbox * NCH * R * 128));
            else mbar_expect_tx(full, (uint32_t)(nbox * NCH * R * 128));
            for (int sb = 0; sb < BLK / R; ++sb) {
                if (pages[sb] < 0) continue;
                const int off = (j * BLK + sb * R) % p.page_size;
#pragma unroll
                for (int c = 0; c < NCH; ++c)
                    tma_load_4d(dst + c * BLK * 128 + sb * R * 128, map, full, c * CH, hk, off,
                                pages[sb]);
            }
        }
    } else {
        const int t = -item - 1;
        if (arrive) mbar_arrive_expect_tx(full, TILE_BYTES);
        else mbar_expect_tx(full, TILE_BYTES);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
            tma_load_3d(dst + c * BLK * 128, mean_map, full, c * CH, t * BLK, b * p.Hkv + hk);
    }
}

// Page ids of the work items are resolved by the whole producer warp, 32
// items at a time (one lane per item), into a ring of kPageRing items x
// kMaxBoxes sub-boxes in shared memory: the issuing lane then reads them from
// shared memory instead of making one dependent page-table load per tile.
constexpr int kPageRing = 64;
constexpr int kMaxBoxes = 8;  // BLK / page_size for page_size >= 16, BLK <= 128

template <int BLK>
__device__ __forceinline__ void fill_page_ring(const KParams& p, const SeqInfo& s, int b,
                                               const int* items, int n_items, int n0, int* ring) {
    const int lane = threadIdx.x & 31;
    const int n = n0 + lane;
    if (p.paged && n < n_items && items[n] >= 0) {
        const int j = items[n];
        const int R = min(p.page_size, BLK);
        int* dst = ring + (n % kPageRing) * kMaxBoxes;
        for (int sb = 0; sb < BLK / R; ++sb) {
            const int tok = j * BLK + sb * R;
            int pg = -1;
            if (tok < s.Lk) {
                pg = p.page_table[(size_t)b * p.max_pages + tok / p.page_size];
                if (pg < 0 || pg >= p.num_pages) {
                    set_error(p.err, kErrBounds, kDetPage);
                    pg = -1;
                }
            }
            dst[sb] = pg;
        }
    }
    __syncwarp();
}

// Both tiles of a work item into one stage, one barrier: the K tile only
// adds its bytes, the V tile adds its bytes and arrives (once per phase).
template <int D, int BLK, bool FP8>
__device__ __forceinline__ void issue_item_loads(const KParams& p, const AttnMaps& maps,
                                                 const SeqInfo& s, int b, int hk, int item,
                                                 const int* pages, uint32_t k_s, uint32_t v_s,
                                                 uint64_t* full) {
    issue_tile_load<D, BLK, FP8>(p, &maps.k, &maps.kb, s, b, hk, item, pages, k_s, full, false);
    issue_tile_load<D, BLK, FP8>(p, &maps.v, &maps.vb, s, b, hk, item, pages, v_s, full, true);
}

// Zeroes rows [nvalid, BLK) of a V tile (NCH chunks of BLK x 128 bytes) with
// `nthr` cooperating threads (index `tid`).  Whole 128-byte rows are zeroed,
// so the swizzle inside a row does not matter.
template <int BLK, int NCH>
__device__ __forceinline__ void zero_v_tail(uint8_t* v_tile, int nvalid, int tid, int nthr) {
    const int units = (BLK - nvalid) * 8;  // 16-byte units per chunk
    for (int c = 0; c < NCH; ++c)
        for (int x16 = tid; x16 < units; x16 += nthr)
            *reinterpret_cast<uint4*>(v_tile + c * BLK * 128 + nvalid * 128 + x16 * 16) =
                make_uint4(0, 0, 0, 0);
}

}  // namespace fp2
