// fp2_attn_pair.cu -- the block-sparse attention kernel: two 128-row tiles
// per CTA share every K/V tile and alternate on the tensor core.
//
// Same result as the single-tile kernel (fp2_attn.cu): for each query row an
// online softmax over the tokens of the kept key blocks plus one pseudo-token
// per dropped block (logit q.kbar/sqrt(d) + ln n_j, value vbar) -- the
// FlashPrefill V2 abstract's sparse operator with PackGQA access and the
// mean correction term.
//
// Work item = (sequence, KV head, query block i, pair index): tile A holds
// tokens [t0, t0+TOK) x G heads, tile B the next TOK tokens (TOK = 128/G).
// Both tiles belong to query block i, so they walk the same list of kept
// blocks and mean tiles, and each K/V tile is loaded once for 256 rows.
// When a query block packs only 128 rows (G x block = 128: G = 1 with block
// 128, G = 2 with block 64) tile A is query block i and tile B block i+1 of
// the same KV head; the CTA walks the union of the two blocks' lists, and
// each tile masks what its own block does not keep (tile A's rows take
// nothing from block i+1, its causal future).
//
// Roles (384 threads = 3 warpgroups; registers rebalanced with setmaxnreg:
// 224 per softmax thread, 56 in the control warpgroup, 384 x 168 in total):
//   warps 0-3  softmax for tile A (thread = row = TMEM lane)
//   warps 4-7  softmax for tile B
//   warp 8     TMA producer of the K ring, warp 10 of the V ring (2 stages
//              each; the two Q tiles are fetched by thread 0 right after the
//              barriers exist)
//   warp 11    idle
//   warp 9     TMEM owner; lane 0 issues the MMAs in the order
//                PV_A(n-1), QK_A(n), PV_B(n-1), QK_B(n)
//              so that while one warpgroup works on its S the tensor core
//              runs the other tile's two products.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384),
// O_B [384,512).  P_X (bf16 pairs or e4m3 quads) is written over the first
// columns of S_X once the softmax has read S_X, and PV_X reads it from TMEM
// (A operand in tensor memory).  QK_X(n+1) is issued after PV_X(n) by the
// same thread; tcgen05.mma operations of one thread execute in issue order,
// so PV_X(n) has read P_X before QK_X(n+1) overwrites it.  The commit that
// signals S_X(n) full also covers PV_X(n-1), so when a softmax thread reads
// S_X(n), O_X is stable and may be rescaled in place.
#include "fp2_attn_common.cuh"

namespace fp2 {

template <int D, int BLK, bool FP8>
struct PairCfg {
    static constexpr int ELT = FP8 ? 1 : 2;
    static constexpr int CH = 128 / ELT;
    static constexpr int NCH = D / CH;
    static constexpr int KSTEP = FP8 ? 32 : 16;
    static constexpr int Q_BYTES = 128 * D * ELT;   // one tile
    static constexpr int KV_BYTES = BLK * D * ELT;
    static constexpr int P_COLS = BLK * ELT / 4;    // 32-bit TMEM columns of one P row
    static constexpr int S = 2;  // ring depth of K and of V
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + S * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + S * KV_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + 256;
    static constexpr int OFF_RING = OFF_MISC + 64;  // page ids of upcoming items
    static constexpr int OFF_ITEMS = OFF_RING + 2 * kPageRing * kMaxBoxes * 4;  // K and V rings
    static_assert(P_COLS % 32 == 0, "P row must be whole 32-column TMEM stores");
    // pairs (of every 4) whose exp2 runs on the FMA pipe instead of MUFU (one
    // measured best for both types; 0, 2 and 3 were slower)
    static constexpr int kEmuPairs = 1;
    // polynomial degree of the FMA-pipe exp2: e4m3 probabilities need less
    static constexpr int kEmuDeg = FP8 ? 2 : 3;
};

// The FMA-pipe exp2 (exp2_sat_poly2) folds its clamp into a saturating FMA;
// its range ends at exponent 8, which the lazy rescale guarantees: every
// exponent is x * sl2 + bias - m_used with the row's maximum at most
// kRescaleLog2 above m_used.
static_assert(kRescaleLog2 <= 8.f, "exp2_sat_poly2 covers exponents up to 8");


// K and V have separate rings: K(n) is free once QK_B(n) has run, V(n) only
// after PV_B(n) -- a full MMA pair later -- so each stream refills as soon as
// its own operand is consumed.
// KV_FULL[n % 2]: step n has landed, K(n) and V(n-1) together (one barrier
// with one arrival per producer warp, so the MMA thread polls once per item
// for both)
enum { PB_KV_FULL = 0, PB_K_EMPTY = 2, PB_V_EMPTY = 4, PB_Q_FULL = 6, PB_S_FULL = 7,
       PB_P_READY = 9, PB_O_FINAL = 11, PB_DRAIN = 13, PB_COUNT = 14 };

template <int D, int BLK, bool FP8>
__global__ void __launch_bounds__(384, 1)
attn_pair_kernel(const KParams p, const __grid_constant__ AttnMaps maps,
                 const uint32_t* __restrict__ kept_bits, __nv_bfloat16* __restrict__ out,
                 int items_cap) {
    using C = PairCfg<D, BLK, FP8>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + C::OFF_Q;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    int* items = reinterpret_cast<int*>(smem + C::OFF_ITEMS);
    uint32_t* sbits = reinterpret_cast<uint32_t*>(items + items_cap);

    const int G = p.G;
    const int TOK = 128 / G;
    // Tiles of one query block (G x block >= 256 packed rows: npair pairs of
    // tiles per block), or, when a block is a single tile (G x block = 128),
    // two adjacent query blocks i, i+1 (xq): they walk the union of their
    // kept lists; a key block only the second keeps is masked out for the first.
    const int npair = BLK / (2 * TOK);
    const bool xq = npair == 0;
    const int units = xq ? (p.qb_n + 1) / 2 : p.qb_n;
    const int per_u = p.num_seqs * p.Hkv * (xq ? 1 : npair);
    const int u = units - 1 - (int)(blockIdx.x / per_u);  // longest first
    const int rem = (int)(blockIdx.x % per_u);
    const int b = rem / (p.Hkv * (xq ? 1 : npair));
    const int hk = xq ? rem % p.Hkv : (rem / npair) % p.Hkv;
    const int pr = xq ? 0 : rem % npair;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t wlim = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;

    SeqInfo s;
    if (!load_seq(p, b, s)) return;
    const int i = p.qb_lo + (xq ? 2 * u : u);  // query block of tile A
    const int i_b = xq ? i + 1 : i;            // query block of tile B
    // whether tile B has rows (xq: block i+1 exists and is in this launch)
    const bool b_ok = !xq || (i_b < s.nqb && i_b < p.qb_lo + p.qb_n);
    // the tiles' first queries (negative inside a partial first query block)
    const int t_a = i * BLK - s.off + pr * 2 * TOK;
    const int t_b = xq ? i_b * BLK - s.off : t_a + TOK;
    if (i >= s.nqb || t_a >= s.Lq || t_a + 2 * TOK <= 0) return;  // no rows here
    const int iabs = s.pb + i;
    const int iabs_b = s.pb + i_b;
    const int iabs_hi = b_ok ? iabs_b : iabs;  // last key block either tile reaches
    const int nw_c = (iabs_hi + 32) / 32;

    if (threadIdx.x == 0) {
        for (int k = 0; k < PB_COUNT; ++k)
            mbar_init(&bars[k], (k == PB_P_READY || k == PB_P_READY + 1) ? 4u  // one per softmax warp
                                : k < PB_K_EMPTY ? 2u : 1u);  // KV_FULL: one arrival per producer
        misc[1] = 0;
        fence_mbar_init();
        // both Q tiles right away: their latency overlaps the kept-bit loads
        // and the item list
        mbar_arrive_expect_tx(&bars[PB_Q_FULL], 2 * C::Q_BYTES);
        for (int x = 0; x < 2; ++x)
            for (int c = 0; c < C::NCH; ++c)
                tma_load_3d(q_s + x * C::Q_BYTES + c * (128 * 128), &maps.q, &bars[PB_Q_FULL],
                            c * C::CH, hk * G, s.q0 + (x ? t_b : t_a));
    }
    if (warp == 9) {
        tmem_alloc(&misc[0], 512);
        tmem_relinquish();
    }
    // kept bits: G rows for tile A's block, then (xq) G rows for tile B's
    load_kept_bits(p, kept_bits, b, hk, i, iabs, nw_c, sbits);
    if (xq && b_ok) load_kept_bits(p, kept_bits, b, hk, i_b, iabs_b, nw_c, sbits + G * nw_c);
    __syncthreads();
    if (warp == 8) {
        const int n = build_items<BLK>(xq && b_ok ? 2 * G : G, iabs_hi, nw_c, sbits, items);
        if (lane == 0) misc[2] = (uint32_t)n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int n_items = (int)misc[2];

    if (warp >= 8) {
      regs_decrease<56>();
      if (warp == 8 || warp == 10) {
        // --------------------------------------------------------- producers ---
        // warp 8 issues the K ring, warp 10 the V ring; each warp resolves
        // the page ids of its own items 32 at a time into its own page ring,
        // and its lane 0 waits and issues.  Step n of the pipeline is K(n)
        // and V(n-1); KV_FULL[n % 2] counts one arrival from each warp per
        // step, each arriving together with the bytes it will land (a warp
        // with no tile at step n -- K at n = n_items, V at n = 0 -- arrives
        // alone), so a phase cannot complete before both warps registered
        // their bytes.  Before arriving at step n >= 2 a warp makes sure
        // step n-2 (same barrier, previous phase) has completed: implied by
        // its EMPTY wait (K(n) waits for QK_B(n-2), V(n-1) for PV_B(n-3),
        // both issued after the MMA thread saw step n-2 complete), and
        // waited for explicitly where no EMPTY wait implies it.
        const bool is_k = warp == 8;
        int* pring = reinterpret_cast<int*>(smem + C::OFF_RING) +
                     (is_k ? 0 : kPageRing * kMaxBoxes);
        const CUtensorMap* map = is_k ? &maps.k : &maps.v;
        const CUtensorMap* mean_map = is_k ? &maps.kb : &maps.vb;
        const uint32_t ring_s = sbase + (is_k ? C::OFF_K : C::OFF_V);
        uint64_t* empty = &bars[is_k ? PB_K_EMPTY : PB_V_EMPTY];
        if (lane == 0) prefetch_tmap(map);
        int last = -1;  // last step at which this warp arrived on KV_FULL
        bool ok = true;
        for (int n = 0; n <= n_items; ++n) {
            const int m = is_k ? n : n - 1;  // the item this warp loads at step n
            const bool has = m >= 0 && m < n_items;
            if (has && m % 32 == 0) fill_page_ring<BLK>(p, s, b, items, n_items, m, pring);
            if (lane == 0) {
                uint64_t* full = &bars[PB_KV_FULL + n % C::S];
                const int st = m & 1;
                const bool implied = has && m >= C::S;  // the EMPTY wait implies step n-2
                if (n >= 2 && !implied &&
                    !mbar_wait(full, ((n - 2) / C::S) & 1, abort_flag, wlim)) {
                    set_error(p.err, kErrTimeout, kDetWaitBase + 8);
                    ok = false;
                } else if (!has) {
                    mbar_arrive(full);
                    last = n;
                } else if (is_k && p.withhold_k_item == m + 1) {
                    ok = false;  // test knob: K(m) is never loaded nor announced
                } else if (m >= C::S && !mbar_wait(&empty[st], ((m - C::S) / C::S) & 1,
                                                   abort_flag, wlim)) {
                    set_error(p.err, kErrTimeout, kDetWaitBase + 0);
                    ok = false;
                } else {
                    issue_tile_load<D, BLK, FP8>(p, map, mean_map, s, b, hk, items[m],
                                                 pring + (m % kPageRing) * kMaxBoxes,
                                                 ring_s + st * C::KV_BYTES, full, true);
                    last = n;
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
        if (lane == 0) {
            // never leave with copies in flight: wait for the phases of the
            // last two steps this warp arrived at.  Its copies of earlier
            // steps landed before it could arrive at these (the step n-2 rule
            // above), and no later phase of either barrier can complete
            // without this warp, so a parity wait cannot see a stale phase.
            // In a normal run both warps arrive at every step and these waits
            // end at once; one that runs out is recorded (after an abort the
            // first error is already there and a partner that stopped early
            // only costs the limit).
            volatile int no_abort = 0;
            bool drained = true;
            for (int n = max(0, last - 1); n <= last; ++n)
                drained &= mbar_wait(&bars[PB_KV_FULL + n % C::S], (n / C::S) & 1, &no_abort, wlim);
            if (is_k) drained &= mbar_wait(&bars[PB_Q_FULL], 0, &no_abort, wlim);
            if (!drained) set_error(p.err, kErrTimeout, kDetWaitBase + 12);
        }
      } else if (warp == 9 && lane == 0) {
        // -------------------------------------------------------------- MMA ---
            constexpr uint32_t fmt = FP8 ? 0u : 1u;
            constexpr uint32_t idesc_qk = make_idesc(fmt, false, 128, BLK);
            constexpr uint32_t idesc_pv = make_idesc(fmt, true, 128, D);
            bool ok = mbar_wait(&bars[PB_Q_FULL], 0, abort_flag, wlim);
            if (!ok) set_error(p.err, kErrTimeout, kDetWaitBase + 1);
            tc_fence_after();
            for (int n = 0; ok && n <= n_items; ++n) {
                const int st = n & 1;
                // K(n) and V(n-1)
                if (!mbar_wait(&bars[PB_KV_FULL + st], (n >> 1) & 1, abort_flag, wlim)) {
                    set_error(p.err, kErrTimeout, kDetWaitBase + 2);
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int x = 0; x < 2; ++x) {
                    if (n >= 1) {
                        const int m = n - 1;
                        if (!mbar_wait(&bars[PB_P_READY + x], m & 1, abort_flag, wlim)) {
                            set_error(p.err, kErrTimeout, kDetWaitBase + 3);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t v_s = sbase + C::OFF_V + (m & 1) * C::KV_BYTES;
                        const uint32_t p_tmem = tmem + x * 128;
                        const uint32_t o_tmem = tmem + 256 + x * 128;
#pragma unroll
                        for (int ks = 0; ks < BLK / C::KSTEP; ++ks) {
                            const uint64_t bd =
                                sw128_desc(v_s + ks * C::KSTEP * 128, BLK * 128, 1024);
                            const uint32_t acc = (m > 0 || ks > 0) ? 1u : 0u;
                            if constexpr (FP8) mma_f8_ts(o_tmem, p_tmem + ks * 8, bd, idesc_pv, acc);
                            else mma_bf16_ts(o_tmem, p_tmem + ks * 8, bd, idesc_pv, acc);
                        }
                        if (x == 1) mma_commit(&bars[PB_V_EMPTY + (m & 1)]);
                        if (m == n_items - 1) mma_commit(&bars[PB_O_FINAL + x]);
                    }
                    if (n < n_items) {
                        const uint32_t k_s = sbase + C::OFF_K + st * C::KV_BYTES;
                        const uint32_t qx = q_s + x * C::Q_BYTES;
                        const uint32_t s_tmem = tmem + x * 128;
#pragma unroll
                        for (int ks = 0; ks < D / C::KSTEP; ++ks) {
                            const int ch = (ks * C::KSTEP) / C::CH;
                            const uint32_t within = (uint32_t)((ks * C::KSTEP) % C::CH) * C::ELT;
                            const uint64_t ad = sw128_desc(qx + ch * (128 * 128) + within, 16, 1024);
                            const uint64_t bd =
                                sw128_desc(k_s + ch * (BLK * 128) + within, 16, 1024);
                            if constexpr (FP8) mma_f8_ss(s_tmem, ad, bd, idesc_qk, ks > 0);
                            else mma_bf16_ss(s_tmem, ad, bd, idesc_qk, ks > 0);
                        }
                        mma_commit(&bars[PB_S_FULL + x]);
                        if (x == 1) mma_commit(&bars[PB_K_EMPTY + st]);
                    }
                }
            }
            mma_commit(&bars[PB_DRAIN]);
            volatile int no_abort = 0;
            mbar_wait(&bars[PB_DRAIN], 0, &no_abort, wlim);
      }
    } else {
        regs_increase<224>();
        // ---------------------------------------------------------- softmax ---
        const int X = warp >> 2;                  // tile
        const int qw = warp & 3;
        const int r = qw * 32 + lane;             // row of the tile == TMEM lane
        const int g = r % G;
        const int t = (X ? t_b : t_a) + r / G;  // query index in the sequence
        const int iabs_x = X && xq ? iabs_b : iabs;  // this tile's diagonal block
        const int h = hk * G + g;
        const bool row_ok = t >= 0 && t < s.Lq && (X == 0 || b_ok);
        const int ppos = s.P + t;
        const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + X * 128;
        const uint32_t o_addr = tmem + lane_off + 256 + X * 128;
        const uint32_t* hb = sbits + ((X && xq ? G : 0) + g) * nw_c;
        float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
        if constexpr (FP8) sl2 *= p.q_scale[h] * p.k_scale[hk];
        const float lb = __log2f((float)BLK);
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int n = 0; n < n_items; ++n) {
            // Which columns of this item the row takes: decided from shared
            // memory before S is waited for, so those loads' latency hides
            // behind the wait.  Masks act on raw scores (the scale sl2 is
            // positive); the bias of a mean tile (log2 n_j) and the running
            // max fold into the one FFMA that feeds exp2:
            //   p = 2^(x * sl2 + (bias - m)).
            const int item = items[n];
            bool live;                  // this row takes part in this item
            float bias = 0.f;
            // a cache quantised per key block: the block's K factor scales its
            // logits (sl2i), its V factor is folded into P before the e4m3
            // rounding as log2 fv in the exponent (lvi <= 0), and the row sum
            // takes the unscaled p (inv_fv).  Mean tiles are in per-head units.
            float sl2i = sl2, lvi = 0.f, inv_fv = 1.f;
            if constexpr (FP8) {
                if (p.kb_fac && item >= 0) {
                    const size_t fi = ((size_t)b * p.nkb_max + item) * p.Hkv + hk;
                    const float fk = __ldg(p.kb_fac + fi), fv = __ldg(p.vb_fac + fi);
                    sl2i = sl2 * fk;
                    lvi = __log2f(fv);
                    inv_fv = 1.f / fv;
                }
            }
            uint32_t dropped[BLK / 32];  // mean tiles: the row's dropped blocks
            if (item >= 0) {
                live = row_ok && ((hb[item >> 5] >> (item & 31)) & 1u);
            } else {
                const int tv = -item - 1;
                bias = lb;
                live = false;
#pragma unroll
                for (int w = 0; w < BLK / 32; ++w) {
                    const int j0 = tv * BLK + w * 32;
                    uint32_t dm = 0u;
                    if (row_ok && j0 < iabs_x) {
                        dm = ~hb[j0 >> 5];
                        const int nvalid = iabs_x - j0;
                        if (nvalid < 32) dm &= (1u << nvalid) - 1u;
                    }
                    dropped[w] = dm;
                    live |= dm != 0u;
                }
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[PB_S_FULL + X], n & 1, abort_flag,
                                                   wlim))) {
                set_error(p.err, kErrTimeout, kDetWaitBase + 4);
                ok = false;
                break;
            }
            tc_fence_after();
            float2 xv[BLK / 2];  // the row's scores as aligned pairs
            float* x = reinterpret_cast<float*>(xv);
#pragma unroll
            for (int c = 0; c < BLK / 32; ++c) tmem_ld32f(s_addr + c * 32, x + c * 32);
            tmem_wait_ld();

            if (item >= 0) {
                if (live && item == iabs_x) {
                    const int lim = ppos - item * BLK;
#pragma unroll
                    for (int c = 0; c < BLK; ++c) x[c] = c <= lim ? x[c] : -INFINITY;
                }
            } else {
#pragma unroll
                for (int w = 0; w < BLK / 32; ++w)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        x[w * 32 + e] = ((dropped[w] >> e) & 1u) ? x[w * 32 + e] : -INFINITY;
            }
            float mx = -INFINITY;
            if (live) {
                float m0 = x[0], m1 = x[1], m2 = x[2], m3 = x[3];
#pragma unroll
                for (int c = 4; c < BLK; c += 8) {
                    m0 = max3f(m0, x[c], x[c + 1]);
                    m1 = max3f(m1, x[c + 2], x[c + 3]);
                    m2 = max3f(m2, x[c + 4], x[c + 5]);
                    if (c + 7 < BLK) m3 = max3f(m3, x[c + 6], x[c + 7]);
                    else m3 = fmaxf(m3, x[c + 6]);
                }
                mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
                if (mx != -INFINITY) mx = fmaf(mx, sl2i, bias);
            }
            float alpha = 1.f;
            bool rescale = false;
            if (m_used == -INFINITY) {
                m_used = mx;
            } else if (mx > m_used + kRescaleLog2) {
                alpha = ex2(m_used - mx);
                m_used = mx;
                rescale = true;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // O_X is stable here (PV_X(n-1) completed before S_X(n) was signalled)
                const float a = rescale ? alpha : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
                    tmem_st32(o_addr + c * 32, o);
                }
            }
            float sum = 0.f;
            {
                // a row that takes no part gets offset -inf: every p is 0
                const float c0 = live ? bias - m_used + lvi : -INFINITY;
                const float2 k2 = make_float2(sl2i, sl2i), c2 = make_float2(c0, c0);
                const float k128 = sl2i * (1.f / 128.f), c128 = (c0 + 120.f) * (1.f / 128.f);
                float2 a0 = make_float2(0.f, 0.f), a1 = a0;
                // of every 4 pairs, the last kEmuPairs go to the FMA pipe
                // (exp2_sat_poly2), the rest to MUFU ex2: the two units share
                // the load
#pragma unroll
                for (int c = 0; c < BLK / 2; c += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (u >= 4 - C::kEmuPairs) {
                            xv[c + u] = exp2_sat_poly2<C::kEmuDeg>(xv[c + u], k128, c128);
                        } else {
                            const float2 e = ffma2(xv[c + u], k2, c2);
                            xv[c + u] = make_float2(ex2(e.x), ex2(e.y));
                        }
                        if (u & 1) a1 = fadd2(a1, xv[c + u]);
                        else a0 = fadd2(a0, xv[c + u]);
                    }
                }
                sum = ((a0.x + a0.y) + (a1.x + a1.y)) * inv_fv;
            }
            l = l * alpha + sum;
            // P_X -> TMEM over S_X
#pragma unroll
            for (int c = 0; c < C::P_COLS / 32; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    if constexpr (FP8) {
                        const float* src = x + (c * 32 + e) * 4;
                        pk[e] = pack_e4m3x4(src[0], src[1], src[2], src[3]);
                    } else {
                        pk[e] = pack_bf16x2(x[(c * 32 + e) * 2], x[(c * 32 + e) * 2 + 1]);
                    }
                }
                tmem_st32(s_addr + c * 32, pk);
            }
            if (X == 0 && item >= 0 && item * BLK + BLK > s.Lk) {
                // V(n) loads one step behind K(n): let it land before zeroing
                // (V(n+2) cannot reuse the slot before this warpgroup's P(n))
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[PB_KV_FULL + ((n + 1) & 1)], ((n + 1) >> 1) & 1,
                                                       abort_flag, wlim))) {
                    set_error(p.err, kErrTimeout, kDetWaitBase + 7);
                    ok = false;
                    break;
                }
                zero_v_tail<BLK, C::NCH>(smem + C::OFF_V + (n & 1) * C::KV_BYTES,
                                         max(0, s.Lk - item * BLK), r, 128);
                fence_proxy_async_smem();
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();  // the warp's P stores (and V zeroing) before its one arrival
            if (lane == 0) mbar_arrive(&bars[PB_P_READY + X]);
        }
        if (ok && __all_sync(0xffffffffu, mbar_wait(&bars[PB_O_FINAL + X], 0, abort_flag,
                                                    wlim))) {
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
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int BLK, bool FP8>
cudaError_t launch_attn_pair_t(const KParams& p, const void* q, const void* k, const void* v,
                               const uint32_t* kept_bits, void* out, cudaStream_t st) {
    using C = PairCfg<D, BLK, FP8>;
    AttnMaps maps;
    const int TOK = 128 / p.G;
    if (!make_attn_maps(p, q, k, v, D, BLK, TOK, &maps)) return cudaErrorInvalidValue;
    const int items_cap = p.nkb_max + (p.nkb_max + BLK - 1) / BLK + 2;
    const int nw_c_max = p.nkb_max / 32 + 1;
    const bool xq = BLK < 2 * TOK;  // tiles are adjacent query blocks: twice the kept bits
    size_t smem = 1024 + C::OFF_ITEMS + (size_t)items_cap * 4 +
                  (size_t)(xq ? 2 : 1) * p.G * nw_c_max * 4;
    if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM: it owns all 512 TMEM columns
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel<D, BLK, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int npair = BLK / (2 * TOK);
    const long long grid = xq ? (long long)((p.qb_n + 1) / 2) * p.num_seqs * p.Hkv
                              : (long long)p.qb_n * p.num_seqs * p.Hkv * npair;
    if (grid <= 0) return cudaSuccess;
    attn_pair_kernel<D, BLK, FP8><<<(unsigned)grid, 384, smem, st>>>(
        p, maps, kept_bits, static_cast<__nv_bfloat16*>(out), items_cap);
    return cudaGetLastError();
}

cudaError_t launch_attn_pair(const KParams& p, const void* q, const void* k, const void* v,
                             const uint32_t* kept_bits, void* out, cudaStream_t st) {
    if (p.fp8) {
        if (p.d == 128 && p.B == 128) return launch_attn_pair_t<128, 128, true>(p, q, k, v, kept_bits, out, st);
        return cudaErrorInvalidValue;
    }
    if (p.d == 128 && p.B == 128) return launch_attn_pair_t<128, 128, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 128 && p.B == 64) return launch_attn_pair_t<128, 64, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 64 && p.B == 128) return launch_attn_pair_t<64, 128, false>(p, q, k, v, kept_bits, out, st);
    if (p.d == 64 && p.B == 64) return launch_attn_pair_t<64, 64, false>(p, q, k, v, kept_bits, out, st);
    return cudaErrorInvalidValue;
}

}  // namespace fp2
