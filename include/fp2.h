/*
 * fp2.h -- C ABI of the B200 (sm_100a) block-sparse causal prefill attention
 * with block-mean correction (FlashPrefill V2).
 *
 * The method (FlashPrefill V2 abstract, chatpaper.ai card, English abstract;
 * popular explainer, papers.ananclaw.com, sections 2.1-2.3):
 *   1. block means kbar_j, vbar_j of K and V per KV head       (fp2_blockmean)
 *   2. pooled query blocks scored against every causal key
 *      block ("instantaneous pattern discovery")                (fp2_score)
 *   3. max-based dynamic threshold: keep j iff
 *      s_ij >= max_j' s_ij' - tau; block 0 and the diagonal
 *      block are always kept                                    (fp2_mask)
 *   4. online-softmax attention over the kept blocks, GQA heads
 *      packed so a K/V tile is loaded once per group (PackGQA),
 *      plus the mean correction: every dropped block j enters
 *      the same softmax as one pseudo-token with weight
 *      n_j * exp(q.kbar_j / sqrt(d)) and value vbar_j          (fp2_attn)
 * fp2_prefill runs the four in order on one stream.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer unless its comment says host.
 *    The caller owns every buffer; the library never allocates, frees or
 *    synchronises on these calls: all work is enqueued on params->stream
 *    (a cudaStream_t; NULL = the legacy default stream) and the call returns
 *    before it runs.
 *  - q and out are [total_q, Hq, d], row-major, sequences packed by
 *    cu_seqlens (int32 [num_seqs+1], device, cu_seqlens[0] = 0).
 *  - Contiguous K/V (page_table == NULL): k_cache, v_cache are
 *    [total_k, Hkv, d] packed by params->cu_seqlens_k (or by cu_seqlens when
 *    that is NULL).  Paged K/V: [num_pages, page_size, Hkv, d] with
 *    page_table int32 [num_seqs, max_pages_per_seq] of physical page ids.
 *  - Sequence b has Lq = cu_seqlens[b+1]-cu_seqlens[b] new tokens and
 *    Lk = seqlens_k[b] (or Lq when seqlens_k is NULL) keys; query t sits at
 *    absolute position P + t, P = Lk - Lq (the resident prefix, any length:
 *    a decode row is a sequence with Lq = 1).  Query blocks are cut at
 *    absolute positions, like key blocks: query block i of sequence b is
 *    absolute block P/B + i and holds the rows t with (P + t)/B = P/B + i, so
 *    when P is not a multiple of B the first one is partial (explainer
 *    section 2.3: a chunk may mix prefill and decode rows).
 *  - dtype FP2_BF16: q/k/v are bf16.  FP2_FP8_E4M3: q/k/v are e4m3 with
 *    per-head dequantisation scales (x = e4m3 * scale), params->q_scale [Hq],
 *    k_scale [Hkv], v_scale [Hkv] (fp32, device).  out is bf16 unless
 *    params->out_dtype asks for e4m3.
 *  - Base pointers of q, k_cache, v_cache and out must be 16-byte aligned.
 *  - Supported: head_dim 64 or 128, block 64 or 128 (FP8: head_dim 128
 *    and block 128 only; other FP8 shapes return FP2_ERR_UNSUPPORTED),
 *    G = Hq/Hkv in {1,2,4,8} with 128/G <= block, page_size a power of two
 *    in [16, 256] that divides the block or is divided by it.
 *
 * Kernel choice: the two-tile attention kernel runs every problem (two
 * 128-row tiles of one query block when G * block >= 256, else two adjacent
 * query blocks); params->attn_kernel = 1 selects the one-tile kernel instead
 * (a second, independent implementation of the same step, kept for tests).
 *
 * Errors: argument errors are returned synchronously before any launch.
 * CUDA launch errors return FP2_ERR_CUDA.  Problems only the device can see
 * (Lk < Lq, a length above
 * max_seqlen_*, a page id outside [0, num_pages), a bounded wait that ran
 * out) set an error word in the workspace and make the affected blocks skip
 * their work; fp2_get_status reads it.  Nothing prints, nothing throws.
 */
#ifndef FP2_H
#define FP2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP2_OK = 0,
    FP2_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent shapes */
    FP2_ERR_UNSUPPORTED = 2,   /* valid but outside the supported set above */
    FP2_ERR_WORKSPACE = 3,     /* workspace missing or smaller than fp2_workspace_size */
    FP2_ERR_CUDA = 4,          /* a CUDA call failed */
    FP2_ERR_TIMEOUT = 5,       /* device: a bounded pipeline wait ran out */
    FP2_ERR_DEVICE_BOUNDS = 6  /* device: an index (page id, length) out of range */
} fp2_status;

typedef enum { FP2_BF16 = 0, FP2_FP8_E4M3 = 1 } fp2_dtype;

typedef struct fp2_params {
    int num_seqs;              /* >= 1 */
    int num_q_heads;           /* Hq */
    int num_kv_heads;          /* Hkv, divides Hq */
    int head_dim;              /* d */
    int total_q;               /* rows of q and out */
    int total_k;               /* contiguous K/V: rows of k_cache/v_cache; paged: 0 */
    int page_size;             /* paged only: tokens per page */
    int max_pages_per_seq;     /* paged only: row stride of page_table */
    int num_pages;             /* paged only: pages in k_cache/v_cache */
    int max_seqlen_q;          /* >= every Lq; sizes the workspace */
    int max_seqlen_k;          /* >= every Lk; sizes the workspace */
    const int32_t* seqlens_k;  /* device [num_seqs] or NULL (Lk = Lq) */
    const int32_t* cu_seqlens_k; /* device [num_seqs+1], contiguous K/V only, or NULL */
    const float* q_scale;      /* FP8 only, device [Hq] */
    const float* k_scale;      /* FP8 only, device [Hkv] */
    const float* v_scale;      /* FP8 only, device [Hkv] */
    void* workspace;           /* device, fp2_workspace_size() bytes, 256-byte aligned */
    size_t workspace_bytes;
    void* stream;              /* cudaStream_t */
    int group_masks;           /* 0 (default): one mask per query head.  1: one mask per KV
                                  group (a variant): fp2_score scores every head of a group
                                  with the group-mean pooled query, so all G heads keep the
                                  same blocks and PackGQA walks no union of differing lists */
    int out_dtype;             /* FP2_BF16 (default): out is bf16.  FP2_FP8_E4M3: out is e4m3
                                  [total_q, Hq, d] holding O / out_scale[h], saturating */
    const float* out_scale;    /* device [Hq], e4m3 output only.  NULL with FP8 inputs: the
                                  KV head's v_scale (|O| <= max|V|, so it never saturates);
                                  required with BF16 inputs */
    int attn_kernel;           /* 0 (default): the two-tile attention kernel.  1: the one-tile
                                  kernel (same results within rounding; for tests) */
    unsigned int debug_wait_limit_us; /* 0 (default): every pipeline wait inside the
                                  attention kernel gives up after 2 s, records
                                  FP2_ERR_TIMEOUT and ends its CTA cleanly.  > 0: after this
                                  many microseconds instead (tests of that path) */
    int debug_withhold_k_item; /* 0 (default).  > 0, tests only: the two-tile kernel's
                                  producer never loads the K tile of that work item
                                  (1-based) in any CTA, so the consumer's bounded wait runs
                                  out and the call records FP2_ERR_TIMEOUT; the output is
                                  then undefined.  Never set in normal use */
    const float* k_block_factor; /* e4m3 only, optional (NULL: one scale per head): a KV
                                  cache quantised per key block.  Device fp32
                                  [num_seqs][ceil(max_seqlen_k / block)][Hkv]: key block j of
                                  sequence b, KV head h dequantises as
                                  x = e4m3 * k_scale[h] * k_block_factor[b][j][h], factor in
                                  (0, 1] (k_scale[h] is then the head's largest block scale).
                                  A factor outside (0, 1] records FP2_ERR_INVALID_ARG
                                  (detail 5) on the device.  Given together with
                                  v_block_factor; the two-tile attention kernel only */
    const float* v_block_factor; /* the same for V */
} fp2_params;

/* Offsets (bytes from params->workspace) of the intermediates, for callers
 * that read them (parity checks, exported masks).  Per-sequence regions are
 * padded to nqb_max = min(floor((max_seqlen_q + 2B - 2)/B), nkb_max) query
 * blocks (one more than ceil(max_seqlen_q/B) when a prefix that is not a
 * multiple of B can shift a sequence's queries across a block boundary) and
 * nkb_max = ceil(max_seqlen_k/B) key blocks; nw = ceil(nkb_max/32). */
typedef struct fp2_workspace_layout {
    size_t error_word;  /* uint32 [4]: first error code, detail */
    size_t kbar;        /* fp32 [num_seqs][Hkv][nkb_max][d]: dequantised key block means */
    size_t vbar;        /* fp32 [num_seqs][Hkv][nkb_max][d] */
    size_t kbar_op;     /* bf16|e4m3 [num_seqs][Hkv][nkb_max][d]: means as MMA operands */
    size_t vbar_op;     /* (FP8: in the units of k_scale / v_scale) */
    size_t scores;      /* fp32 [num_seqs][Hq][nqb_max][nkb_max], j <= i_abs written */
    size_t kept_idx;    /* int32 [num_seqs][Hq][nqb_max][nkb_max], ascending kept j */
    size_t kept_cnt;    /* int32 [num_seqs][Hq][nqb_max] */
    size_t kept_bits;   /* uint32 [num_seqs][Hq][nqb_max][nw], bit j = block j kept */
    size_t total;       /* bytes needed */
    int nqb_max, nkb_max, nw;
} fp2_workspace_layout;

/* Workspace bytes for these params and block size (0 on invalid params). */
size_t fp2_workspace_size(const fp2_params* params, int block);

/* Fills *layout; FP2_ERR_INVALID_ARG on invalid params. */
fp2_status fp2_get_workspace_layout(const fp2_params* params, int block,
                                    fp2_workspace_layout* layout);

/* The whole path: blockmean -> score -> mask -> attn.  tau >= 0 or +inf is
 * the usual range (any non-NaN value is accepted; tau = +inf keeps every
 * block and gives exact causal attention).  out: bf16 [total_q, Hq, d]. */
fp2_status fp2_prefill(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* page_table, const int32_t* cu_seqlens,
                       float tau, int block, fp2_dtype dtype, void* out,
                       const fp2_params* params);

/* fp2_prefill with step 1 served by the block-mean cache (fp2_blockmean_cached). */
fp2_status fp2_prefill_cached(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* page_table, const int32_t* cu_seqlens, float tau,
                              int block, fp2_dtype dtype, void* out, const fp2_params* params,
                              const int32_t* block_table, int max_blocks_per_seq,
                              float* mean_cache, int num_slots);

/* Step 1 (explainer section 2.1, the mean of the dropped tokens): block means
 * of K and V into the workspace (kbar, vbar, kbar_op, vbar_op); key blocks
 * beyond a sequence's end are written as zeros. */
fp2_status fp2_blockmean(const void* k_cache, const void* v_cache, const int32_t* page_table,
                         const int32_t* cu_seqlens, int block, fp2_dtype dtype,
                         const fp2_params* params);

/* Step 1 for a chunked prefill over a resident prefix, with a block-mean
 * cache kept beside the paged KV cache (so a new chunk does not re-read the
 * whole prefix to average it).  The cache is caller-owned device memory,
 * mean_cache fp32 [num_slots][2][Hkv][d]: per slot the means of the STORED
 * K values, then of the stored V values, of one key block (before any FP8
 * scale).  block_table int32 [num_seqs][max_blocks_per_seq] (device) gives
 * the slot of key block j of sequence b.  Blocks wholly inside the prefix
 * (j*block + block <= Lk - Lq) are read from their slot; every other block of
 * the sequence is averaged from k_cache/v_cache and ALSO written to its slot
 * (so the next chunk finds it).  The workspace receives exactly what
 * fp2_blockmean would write.  A slot id outside [0, num_slots) or a block
 * beyond max_blocks_per_seq records FP2_ERR_DEVICE_BOUNDS (detail 4).
 * mean_cache must be 16-byte aligned. */
fp2_status fp2_blockmean_cached(const void* k_cache, const void* v_cache,
                                const int32_t* page_table, const int32_t* cu_seqlens,
                                const int32_t* block_table, int max_blocks_per_seq,
                                float* mean_cache, int num_slots, int block, fp2_dtype dtype,
                                const fp2_params* params);

/* Step 2 (abstract: instantaneous pattern discovery): pools each query block
 * (mean of the sequence's rows inside it; the first block of a sequence whose
 * prefix is not a multiple of B holds only the rows from P on) and writes s_ij = qbar_i . kbar_j / sqrt(d) for
 * every causal j into the workspace scores.  Needs step 1. */
fp2_status fp2_score(const void* q, const int32_t* cu_seqlens, int block, fp2_dtype dtype,
                     const fp2_params* params);

/* Step 3 (abstract: max-based dynamic thresholding): writes kept_idx,
 * kept_cnt and kept_bits into the workspace.  Needs step 2. */
fp2_status fp2_mask(const int32_t* cu_seqlens, float tau, int block, const fp2_params* params);

/* Step 4 (abstract: sparse operator with PackGQA, warp specialisation and
 * pipelining; the mean correction term): tcgen05/TMEM attention over the
 * blocks set in kept_bits (uint32 [num_seqs][Hq][nqb_max][nw], the layout of
 * the workspace's kept_bits; pass NULL to use the workspace's own), with the
 * block-mean pseudo-tokens for every causal block that is not set.  Needs
 * step 1 (the means).  Bits for j > i_abs are ignored; block 0 and the
 * diagonal are treated as set whatever the bits say. */
fp2_status fp2_attn(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* page_table, const int32_t* cu_seqlens,
                    const uint32_t* kept_bits, int block, fp2_dtype dtype, void* out,
                    const fp2_params* params);

/* Zeroes the workspace's error word (asynchronously, on params->stream).
 * Call it once on a new workspace before the first call that uses it; after
 * that fp2_get_status keeps it clear. */
fp2_status fp2_workspace_init(const fp2_params* params);

/* Synchronises params->stream, returns the first device-side error recorded
 * in the workspace since the last call (FP2_OK if none) and clears it.
 * detail (host, may be NULL) receives the error's detail word. */
fp2_status fp2_get_status(const fp2_params* params, uint32_t* detail);

/* Host utility, not on the hot path (synchronises): the tau at which the
 * scores in the workspace (after fp2_score) drop target_drop of all causal
 * block pairs (forced blocks counted as kept): the midpoint of the two
 * adjacent margins max_j' s_ij' - s_ij at that quantile.  *tau_out is host. */
fp2_status fp2_calibrate_tau(const int32_t* cu_seqlens, int block, float target_drop,
                             const fp2_params* params, float* tau_out);

/* Host-resident inputs and outputs of fp2_prefill_host.  Every pointer is
 * caller-owned; the library allocates nothing.  Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister): pageable memory works but its copies do
 * not overlap the kernels. */
typedef struct fp2_host_io {
    const void* q_host;   /* [total_q, Hq, d] q (bf16 or e4m3, as dtype) */
    const void* k_host;   /* the whole K cache, the layout k_cache has in fp2_prefill:
                             [total_k, Hkv, d] or [num_pages, page_size, Hkv, d] */
    const void* v_host;   /* the whole V cache, same layout */
    void* out_host;       /* [total_q, Hq, d], bf16 or e4m3 (params->out_dtype) */
    void* q_dev;          /* device buffers of the same sizes, 16-byte aligned */
    void* k_dev;
    void* v_dev;
    void* out_dev;
    const int32_t* cu_seqlens_host; /* host copy of cu_seqlens [num_seqs+1] */
    const int32_t* seqlens_k_host;  /* host copy of params->seqlens_k [num_seqs],
                                       NULL when params->seqlens_k is NULL */
    const int32_t* cu_seqlens_k_host; /* host copy of params->cu_seqlens_k [num_seqs+1],
                                       NULL when that is NULL (contiguous K/V only) */
    void* upload_stream;   /* cudaStream_t for the host->device copies; NULL:
                              params->stream (no overlap) */
    void* download_stream; /* cudaStream_t for the device->host copies; NULL:
                              params->stream (no overlap) */
    int num_chunks;        /* query-block chunks of the pipeline, 1..64 */
} fp2_host_io;

/* fp2_prefill with q, K/V and out in host memory: the call a serving process
 * makes when the layer's inputs are not yet on the GPU (packaging of the
 * same method, not a step of it).  It runs block means, score, mask and
 * attention over num_chunks ranges of query blocks, lowest first, uploading
 * each range's query rows (and, for contiguous K/V, the key blocks it adds)
 * while the previous range computes, and downloading each range's output
 * rows while the next one computes; a paged cache is uploaded whole first.
 * Results are bit-identical to fp2_prefill on the same data.
 *  - Queues work on params->stream, io->upload_stream and
 *    io->download_stream and returns; params->stream is made to wait for the
 *    last download, so synchronising params->stream means out_host is done.
 *    The uploads first wait for work already queued on params->stream, so
 *    back-to-back calls on the same device buffers do not race.
 *  - cu_seqlens, params->seqlens_k, params->cu_seqlens_k and page_table
 *    stay device arrays (small, usually resident); the *_host copies must
 *    hold the same values (they place each range's rows).
 *  - Uses a library-owned pool of CUDA events per device, created on the
 *    first call (make it before any stream capture); calls from several
 *    host threads are serialised while they queue.
 *  - Errors as fp2_prefill; io == NULL, a NULL buffer, num_chunks outside
 *    [1, 64] or misaligned device buffers return FP2_ERR_INVALID_ARG. */
fp2_status fp2_prefill_host(const fp2_host_io* io, const int32_t* page_table,
                            const int32_t* cu_seqlens, float tau, int block, fp2_dtype dtype,
                            const fp2_params* params);

/* Bytes of the library-owned device scratch used by fp2_prefill_noalloc. */
#define FP2_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* fp2_prefill for callers that cannot allocate device memory.  The paper has
 * no counterpart: this is a packaging variant, not a step of the method.
 * Plugin-style hosts that hand a kernel only its inputs and outputs, and
 * serving runtimes that reserve all device memory up front (so that a
 * cudaMalloc on the request path would fail or stall the device), cannot
 * supply the workspace fp2_prefill needs.  This call takes the same
 * arguments, ignores params->workspace / params->workspace_bytes, and keeps
 * its scratch in a library-owned device array of FP2_NOALLOC_SCRATCH_BYTES
 * (every GPU that loads the library holds it until the process exits).  It
 * allocates nothing.
 *  - A problem whose fp2_workspace_size() exceeds FP2_NOALLOC_SCRATCH_BYTES
 *    (e.g. one 32K-token sequence with 32 query heads fits; 128K does not) is
 *    rejected with FP2_ERR_WORKSPACE before anything is queued.
 *  - The first call on a device looks up the array's device address (a
 *    synchronous runtime query, once per device); make that first call
 *    before any stream capture.
 *  - Every call shares the one array and leaves its contents behind; calls
 *    whose work overlaps on the GPU (other streams, other host threads) race
 *    on it, so the caller must serialise them.
 *  - Arguments are checked exactly as fp2_prefill checks them, before the
 *    array is touched: a rejected call queues nothing.
 *  - The array's error word is cleared at the start of each call; the
 *    device-side errors of the last call are read with
 *    fp2_noalloc_get_status (not fp2_get_status, which reads a caller's
 *    workspace). */
fp2_status fp2_prefill_noalloc(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* page_table, const int32_t* cu_seqlens,
                               float tau, int block, fp2_dtype dtype, void* out,
                               const fp2_params* params);

/* fp2_get_status for fp2_prefill_noalloc: synchronises `stream` (a
 * cudaStream_t; NULL = the legacy default stream) and returns the first
 * device-side error recorded in the library-owned array of the current device
 * since it was last cleared (FP2_OK if none), then clears it.  *detail (host,
 * may be NULL) receives the error's detail word.  The paper has no
 * counterpart; packaging, like fp2_prefill_noalloc itself. */
fp2_status fp2_noalloc_get_status(void* stream, uint32_t* detail);

/* Static string naming a status code. */
const char* fp2_status_string(fp2_status status);

/* Library version, "major.minor.patch". */
const char* fp2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP2_H */
