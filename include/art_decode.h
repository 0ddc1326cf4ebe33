/*
 * art_decode.h -- C ABI of the B200 (sm_100a) decode-attention library with
 * ART (runtime attention termination) and the q8 V-dequantisation skip.
 *
 * What it computes (web pages, cited by title and section):
 *   "Resumen Tecnico: ART (Terminacion de la Atencion en Tiempo de Ejecucion)",
 *   gist.science summary of arXiv 2606.00024:
 *     S1   one decode query per head attends to the whole cached K/V;
 *     S2.1 attention is accumulated tile by tile (online softmax), which
 *          exposes the partial output O^(t) after every KV tile;
 *     S2.2 ART watches a probe x^(t) (fixed lanes of O^(t)) and stops reading
 *          KV tiles once both its magnitude change d_scale and its direction
 *          change d_direction fall below the thresholds;
 *     S2.3 the criterion must hold on `patience` consecutive tiles;
 *     S2.4 tile 0 is always processed before any termination.
 *   "La paradoja de la eficiencia: como omitir redefine la velocidad de los
 *   LLM", puntofijo.es, section "La Elegancia de la Omision": with an int8
 *   (q8_0) cache the V rows whose softmax weight is negligible are not
 *   dequantised.
 *
 * Readings this library implements (the pages leave them open):
 *   d_scale   = | ||x^(t)|| - ||x^(t-1)|| |
 *   d_dir     = 1 - cos(x^(t), x^(t-1)), >= 0; 0 if both probes are zero,
 *               1 if exactly one is; the probe before a split's first tile is
 *               the zero vector (so +inf thresholds stop after one tile);
 *   hold      = d_scale < eps_scale && d_dir < eps_dir (strict; NaN never holds);
 *   the rule runs per (batch, query head) and independently per KV split;
 *   a head whose rule fires keeps the state of its stop tile; the KV head's
 *   reads stop when all of its query heads have stopped;
 *   split s covers tiles [floor(s*n/S), floor((s+1)*n/S)), n = ceil(L_b/T);
 *   V skip: a row is left out of the numerator when exp(s_j - m') < tau, m'
 *   the running maximum of the split after the row's tile; its weight stays
 *   in the denominator.
 *
 * Conventions for every entry point:
 *   - Tensors are caller-owned DEVICE pointers, contiguous, row-major:
 *       q      [B, Hq, d]          fp32 (ART_F32) or bf16 (ART_BF16, q8 mode)
 *       k, v   [B, Hkv, L_max, d]  fp32 / bf16 / int8 codes
 *       k_scale_f16, v_scale_f16   [B, Hkv, L_max, d/32] IEEE fp16 bits (q8)
 *       seq_lens [B] int32, each in [1, L_max] (checked on the device)
 *       o      [B, Hq, d] fp32 output
 *       tiles  [B, Hq] int32 output: KV tiles consumed per query head (summed
 *              over splits); may be NULL
 *     Query head hq reads KV head hq / (Hq/Hkv).  Device pointers must be
 *     16-byte aligned.
 *   - ws is a caller-owned DEVICE workspace of at least
 *     art_workspace_bytes(shape) bytes, zero-filled once before its first use
 *     (it holds a sticky device status word, per-split partial results and
 *     the per-(batch, kv head, split) count of KV tiles actually read).
 *     One workspace must not be used by two calls that overlap in time.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; nothing is synchronised.  The library
 *     allocates no memory and keeps no global state besides cached kernel
 *     attributes.
 *   - Argument errors are returned synchronously and enqueue nothing.  Errors
 *     found on the device (a seq_len outside [1, L_max], a wait that timed
 *     out) set the status word in ws; art_read_device_status() reports and
 *     clears it.  A head whose seq_len is invalid gets NaN outputs and 0 tiles.
 *   - Constraints (else ART_ERR_UNSUPPORTED or ART_ERR_INVALID_ARG):
 *       d in {64, 128}; tile in {16, 32, 64, 128, 256} and small enough that
 *       two K+V tiles fit in shared memory; 1 <= Hq/Hkv <= 8 with Hq % Hkv == 0;
 *       num_splits >= 1; for q8, L_max*(d/32)*2 bytes a multiple of 16;
 *       1 <= n_probe <= 32 distinct lanes in [0, d); patience >= 1.
 */
#ifndef ART_DECODE_H
#define ART_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library is compiled with hidden visibility; only the declarations below are exported.
 * That also keeps two builds of it (the regular and a test build) loaded in one process from
 * sharing internal state, such as a once-per-device flag inside an inline function. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef enum {
  ART_OK = 0,
  ART_ERR_INVALID_ARG = -1, /* a NULL pointer, a negative size, bad lanes ... */
  ART_ERR_UNSUPPORTED = -2, /* valid but outside what the kernels implement */
  ART_ERR_WORKSPACE = -3,   /* ws NULL or smaller than art_workspace_bytes() */
  ART_ERR_CUDA = -4,        /* a CUDA runtime call failed (launch, attribute) */
  ART_ERR_TIMEOUT = -5,     /* device: a bounded wait gave up (status word) */
  ART_ERR_SEQLEN = -6,      /* device: a seq_len outside [1, L_max] (status word) */
  ART_ERR_ORDER = -7,       /* device: a tile_order entry outside its split (status word) */
  ART_ERR_PAGE = -8,        /* device: a block_table entry outside [0, num_pages) (status word) */
  ART_ERR_INDEX = -9        /* device, debug build (-DART_DEBUG) only: an index check of a kernel
                               failed (status word); regular builds never report it */
} art_status;

typedef enum { ART_F32 = 0, ART_BF16 = 1 } art_dtype;

/* Problem shape.  tile = KV positions per tile (T); num_splits = KV splits per
 * sequence (S): each split runs its own online softmax (and its own ART rule)
 * and a combine step merges them. */
typedef struct {
  int32_t B, Hq, Hkv, d, L_max, tile, num_splits;
} art_shape;

/* ART settings (page S2.2, S2.3).  eps_scale is the page's tau (magnitude),
 * eps_dir its phi (direction).  probe_lanes is a HOST array of n_probe lane
 * indices of O; it is copied during the call.
 *
 * max_spec_tiles bounds the reading ahead of the stopping rule (it changes which
 * K/V tiles are read, never the results).  0: no bound -- the kernel reads as far
 * ahead as its pipeline holds.  n > 0: the tensor-core kernel starts reading a
 * round of tiles only when that round begins fewer than n tiles past the split's
 * "safe" point: the number of tiles every head still running must consume before
 * it can stop (tiles decided so far plus, for the head farthest from stopping,
 * patience minus its current run of holding tiles).  Tiles before the safe point
 * are consumed whatever they hold; at most n tiles plus one round past it are read
 * speculatively.  Negative values are rejected.  The CUDA-core kernel (fp32 / q8
 * one-pass / d = 64 / other tiles), whose CTAs read one round ahead of the rule
 * at most, ignores it, and so does q8 ART on the two streaming passes (which
 * reads every tile; ART_Q8_TENSOR_CORE keeps the bound). */
typedef struct {
  float eps_scale;
  float eps_dir;
  int32_t patience;
  const int32_t* probe_lanes;
  int32_t n_probe;
  int32_t max_spec_tiles;
} art_params;

/* Bytes of workspace a call with this shape needs (0 on an invalid shape).  With one split it
 * includes room for full attention to run as up to 4 internal splits of each sequence (same
 * result; chosen by the library when that keeps more SMs busy); the caller-visible arrays below
 * keep the caller's split layout either way. */
size_t art_workspace_bytes(const art_shape* shape);

/* Bytes of workspace art_decode_attn_q8_skipv needs to run as two streaming passes:
 * art_workspace_bytes(shape) plus scores [B, Hkv, L_max, GP] fp32 (GP the next power of two
 * >= Hq/Hkv), tile and chunk maxima, per-chunk partial states and, for ART, a 136-byte probe
 * record per query head and tile and a stop tile per query head and split (0 on an invalid
 * shape).  The offsets below hold for this larger workspace too. */
size_t art_q8_workspace_bytes(const art_shape* shape);

/* Byte offset inside ws of the int32 array tiles_read[B, Hkv, num_splits]:
 * KV tiles actually fetched from HBM for each (batch, kv head, split) by the
 * last call, speculative prefetch included.  Written by every call. */
size_t art_workspace_tiles_read_offset(const art_shape* shape);

/* Byte offset inside a workspace of art_q8_workspace_bytes(shape) bytes of the
 * int32 array vskip[B, Hkv, num_splits][2]: for each (batch, kv head, split),
 * the V rows left out of every query head's numerator by the V skip (page
 * "La Elegancia de la Omision": exp(s_j - m') < tau for every head of the group)
 * and the V tiles not read at all because every row of every head was left out.
 * Written by the two-pass q8 implementation (art_decode_attn_q8_skipv on the
 * two-pass path; with ART, by its probe pass, over every tile) only; other calls
 * leave it untouched. */
size_t art_workspace_vskip_offset(const art_shape* shape);

/* Byte offset inside ws of the int32 array split_tiles[B, Hq, num_splits]:
 * KV tiles consumed by each (batch, query head, split) in the last call (the
 * per-split terms of `tiles`).  Written by every call. */
size_t art_workspace_split_tiles_offset(const art_shape* shape);

/* Plain tile-wise decode attention over every KV position (page S1, S2.1):
 * o = softmax(q K^T / sqrt(d)) V per query head; tiles = ceil(L_b / tile). */
art_status art_decode_attn_full(const art_shape* shape, art_dtype dtype, const void* q,
                                const void* k, const void* v, const int32_t* seq_lens, float* o,
                                int32_t* tiles, void* ws, size_t ws_bytes, void* stream);

/* Decode attention with ART (page S2.2-S2.4): each (query head, split) stops
 * consuming KV tiles once the probe has been stable for `patience` tiles; o is
 * the normalised partial output at the stop tile, tiles the tiles consumed. */
art_status art_decode_attn_terminate(const art_shape* shape, art_dtype dtype, const void* q,
                                     const void* k, const void* v, const int32_t* seq_lens,
                                     const art_params* params, float* o, int32_t* tiles, void* ws,
                                     size_t ws_bytes, void* stream);

/* Allocation-free variant of art_decode_attn_terminate, for callers that
 * cannot allocate device memory: a host framework that hands a plugin or
 * custom op only its input and output buffers (no workspace argument, no
 * allocator), or code that must not call cudaMalloc on the hot path.  The
 * pages have no counterpart to this entry point; it exists only for those
 * callers.  Same arguments and results as art_decode_attn_terminate, minus
 * ws / ws_bytes: the workspace is a 4 MiB array inside the library
 * (a file-scope __device__ variable, held on every GPU that loads the
 * library until the process exits).
 *   - Shapes whose art_workspace_bytes() exceeds 4 MiB (4194304 bytes) are
 *     rejected with ART_ERR_WORKSPACE before anything is enqueued.
 *   - Calls no cudaMalloc / cudaFree and no allocating library routine.  The
 *     first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture on that device.  The cached address belongs to the
 *     device's current context: after cudaDeviceReset (or anything else that
 *     destroys and recreates the primary context) the array lives at a new
 *     address and the cache is stale, so do not call this entry point again
 *     in that process after a reset.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind.  No word of it has to start at zero (the kernels write all they
 *     read), so nothing is cleared between calls.  Calls whose executions
 *     overlap on the GPU (different streams, or concurrent host threads) race
 *     on the array: serialise them.
 *   - Device-side errors (a seq_len outside [1, L_max]) show as NaN outputs
 *     and 0 tiles for that sequence; there is no status to read back.  A
 *     bounded wait that gives up inside a kernel (a hung copy; it never
 *     happens in normal operation) is not reported either, and leaves the
 *     outputs of the affected sequences unspecified: callers that must
 *     detect it use art_decode_attn_terminate and art_read_device_status. */
art_status art_decode_attn_terminate_noalloc(const art_shape* shape, art_dtype dtype, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             const art_params* params, float* o, int32_t* tiles,
                                             void* stream);

/* Decode attention over an int8 KV cache in 32-element blocks with one fp16
 * scale each (q8_0 style; value = code * scale), bf16 query.  V rows whose
 * weight exp(s_j - m') is below tau are neither dequantised nor accumulated
 * (puntofijo.es, "La Elegancia de la Omision").  params == NULL runs without
 * ART; otherwise ART as in art_decode_attn_terminate.
 * The library picks one of three implementations (same rule, same outputs within rounding,
 * same counters; a tile counts as read when it was fetched):
 *   - with ws_bytes >= art_q8_workspace_bytes(shape) (and B*Hkv*num_splits <= 65535), two
 *     streaming passes over the whole GPU: scores and tile maxima from K, then the running
 *     maxima m', the skip test and the V products (a tile whose rows all fail the test for
 *     every head is not read), then a combine.  With ART (d = 128, tile >= 32, 3 or 4 query
 *     heads per kv head) the V pass runs twice around the rule: a probe pass records per tile
 *     and head (m'_t, l_t, the probe lanes of the tile's sum), a rule kernel finds each head's
 *     stop tile from those records, and the second pass sums the consumed tiles only.  Every
 *     K tile is read (tiles read = all tiles) and max_spec_tiles does not apply;
 *   - otherwise on the tensor cores when d = 128, 3 or 4 query heads per kv head, tile 64 or
 *     128 and L_max even: int8 codes become f16 MMA operands exactly, the scores take the K
 *     scales per 32-element block in fp32, the V scales are folded into the weights, and the
 *     running maxima m' of the V skip are exchanged between the CTAs of a cluster every round;
 *   - otherwise one pass on the CUDA cores that deals the tiles of a split over a
 *     thread-block cluster and exchanges tile maxima every round. */
art_status art_decode_attn_q8_skipv(const art_shape* shape, const void* q_bf16, const int8_t* k_q,
                                    const uint16_t* k_scale_f16, const int8_t* v_q,
                                    const uint16_t* v_scale_f16, const int32_t* seq_lens,
                                    float tau, const art_params* params, float* o, int32_t* tiles,
                                    void* ws, size_t ws_bytes, void* stream);

/* Implementations of art_decode_attn_q8_skipv, for art_decode_attn_q8_skipv_path. */
typedef enum {
  ART_Q8_AUTO = 0,         /* the library's choice (as art_decode_attn_q8_skipv) */
  ART_Q8_TENSOR_CORE = 1,  /* tcgen05 tensor cores */
  ART_Q8_TWO_PASS = 2,     /* two streaming passes + combine (q8 workspace; ART: + probe pass and rule) */
  ART_Q8_CLUSTER = 3       /* one pass on the CUDA cores over a thread-block cluster */
} art_q8_path;

/* art_decode_attn_q8_skipv on a named implementation (testing, benchmarking, or pinning one
 * kernel in production).  Same arguments, plus `path`; ART_ERR_UNSUPPORTED (nothing enqueued)
 * when that implementation does not take the shape or mode (see art_decode_attn_q8_skipv),
 * ART_ERR_INVALID_ARG for an unknown path. */
art_status art_decode_attn_q8_skipv_path(const art_shape* shape, const void* q_bf16, const int8_t* k_q,
                                         const uint16_t* k_scale_f16, const int8_t* v_q,
                                         const uint16_t* v_scale_f16, const int32_t* seq_lens, float tau,
                                         const art_params* params, float* o, int32_t* tiles, void* ws,
                                         size_t ws_bytes, int32_t path, void* stream);

/* ---- KV tile traversal orders ("Resumen Tecnico: ART", S2.4: ART composes with
 * other KV-cache policies by reordering the traversal sequence of the KV blocks,
 * "recency first" or "importance first"; reordering does not change full
 * attention; block 0 comes first).  The page names the orders without defining
 * them; this library's readings:
 *   - A traversal sequence is an int32 array tile_order[B, Hkv, n_max],
 *     n_max = ceil(L_max / tile), DEVICE memory, one sequence per (batch, kv
 *     head).  With num_splits = S, split s of a sequence of n = ceil(L_b/tile)
 *     tiles walks positions [floor(s*n/S), floor((s+1)*n/S)), and those
 *     positions must hold a permutation of split s's own tiles (the same
 *     index range).  Positions >= n are ignored (the builders write -1).
 *   - recency first: each split's first tile, then its other tiles from the
 *     newest back to the oldest.
 *   - importance first: each split's first tile, then its other tiles by the
 *     score max over the kv head's query heads g of q_g . mu_t (mu_t the mean
 *     key of tile t, art_tile_key_summary), highest first, ties to the lower
 *     tile index; scores are computed in fp32.
 * The builders read seq_lens on the device; a sequence whose seq_len is
 * outside [1, L_max] gets -1 everywhere.  They allocate nothing and only
 * enqueue work on `stream`. */

/* Recency-first sequences for every (batch, kv head) into tile_order. */
art_status art_tile_order_recency(const art_shape* shape, const int32_t* seq_lens, int32_t* tile_order,
                                  void* stream);

/* Per-tile key summary: summary[B, Hkv, n_max, d] fp32 (DEVICE) = mean of K over
 * each tile's positions [t*tile, min((t+1)*tile, L_b)); 0 for tiles past L_b.
 * k as in the decode calls (fp32 or bf16, [B, Hkv, L_max, d]); d in {64, 128}. */
art_status art_tile_key_summary(const art_shape* shape, art_dtype dtype, const void* k, const int32_t* seq_lens,
                                float* summary, void* stream);

/* Importance-first sequences from the query q[B, Hq, d] (fp32 or bf16) and a
 * key summary.  One thread block per (batch, kv head) holds n_max scores in
 * shared memory: shapes needing more than 200 KiB give ART_ERR_UNSUPPORTED. */
art_status art_tile_order_importance(const art_shape* shape, art_dtype dtype, const void* q, const float* summary,
                                     const int32_t* seq_lens, int32_t* tile_order, void* stream);

/* Decode attention with ART along caller-given traversal sequences ("Resumen
 * Tecnico: ART", S2.2-S2.4): as art_decode_attn_terminate, but split s of each
 * (batch, kv head) consumes the tiles listed at its positions of tile_order, in
 * that order, and the rule watches the probe along that sequence; `tiles` and the
 * per-split counters count tiles consumed.  With both thresholds 0 it is full
 * attention in any order.  tile_order is DEVICE memory (4-byte aligned).  An
 * entry outside its split is replaced by the natural tile at that position and
 * flags ART_ERR_ORDER in the status word (results of that call are then
 * unspecified); duplicate entries inside the split's range are not detected. */
art_status art_decode_attn_terminate_ordered(const art_shape* shape, art_dtype dtype, const void* q,
                                             const void* k, const void* v, const int32_t* seq_lens,
                                             const art_params* params, const int32_t* tile_order, float* o,
                                             int32_t* tiles, void* ws, size_t ws_bytes, void* stream);

/* ---- Paged KV cache.  The serving stack the pages measure against (vLLM; the
 * intelligenzai.it page on random-attention eviction quotes its step latencies on an
 * H200) keeps the cache in fixed-size pages behind a per-sequence block table.  Position j of
 * sequence b lives in page block_table[b][j / page_size], row j % page_size, of
 * page pools laid out [num_pages][Hkv][page_size][d] (q8 scales
 * [num_pages][Hkv][page_size][d/32]).  Pages may be shared between sequences.
 * Entries of a block-table row past ceil(L_b / page_size) are never read.  An
 * entry outside [0, num_pages) is replaced by page 0 and flags ART_ERR_PAGE in
 * the status word (results of that call are then unspecified). */
typedef struct {
  int32_t page_size;         /* positions per page: a multiple of shape->tile (the tensor-core
                                kernel needs a multiple of 64; others use the CUDA-core kernel) */
  int32_t num_pages;         /* pages in each pool */
  int32_t max_pages_per_seq; /* columns of block_table; shape->L_max <= max_pages_per_seq * page_size */
  const int32_t* block_table; /* DEVICE int32 [B][max_pages_per_seq] */
} art_paged_kv;

/* Decode attention over a paged cache: full attention (params == NULL) or ART
 * (params != NULL), optionally along traversal sequences (tile_order != NULL,
 * ART only; see art_decode_attn_terminate_ordered).  Same outputs, workspace and
 * errors as the contiguous entry points; k_pages / v_pages are the pools. */
art_status art_decode_attn_paged(const art_shape* shape, art_dtype dtype, const void* q, const void* k_pages,
                                 const void* v_pages, const art_paged_kv* pages, const int32_t* seq_lens,
                                 const art_params* params, const int32_t* tile_order, float* o, int32_t* tiles,
                                 void* ws, size_t ws_bytes, void* stream);

/* art_decode_attn_q8_skipv over a paged q8 cache (pools of int8 codes and fp16
 * scales); params == NULL runs without ART. */
art_status art_decode_attn_q8_skipv_paged(const art_shape* shape, const void* q_bf16, const int8_t* k_q_pages,
                                          const uint16_t* k_scale_pages, const int8_t* v_q_pages,
                                          const uint16_t* v_scale_pages, const art_paged_kv* pages,
                                          const int32_t* seq_lens, float tau, const art_params* params, float* o,
                                          int32_t* tiles, void* ws, size_t ws_bytes, void* stream);

/* ---- Random KV eviction ahead of ART (intelligenzai.it page on arXiv 2609.03430,
 * Random Attention: keep the initial prompt and the most recent window, drop the
 * rest uniformly at random inside each head; "Resumen Tecnico: ART" S2.4: ART runs
 * on what a cache policy keeps).  This library's reading, per (batch, kv head):
 * a sequence of length L <= budget keeps every position; otherwise it keeps
 * [0, n_sink), [L - n_recent, L) and the m = budget - n_sink - n_recent middle
 * positions j whose (rand_keys[b][h][j], j) pairs are the m smallest (a uniform
 * draw without replacement when the keys are uniform and independent).  The
 * caller supplies the random keys, so the draw is reproducible.  The kept rows
 * are then packed (art_evict_compact) into a cache of L_max = budget, and any
 * decode entry point runs on it with seq_lens = kept_lens. */
typedef enum { ART_KV_F32 = 0, ART_KV_BF16 = 1, ART_KV_Q8 = 2 } art_kv_format;

/* kept[B][Hkv][budget] int32 (DEVICE): the kept positions in increasing order,
 * -1 past min(L_b, budget); kept_lens[B] (DEVICE) = min(L_b, budget) (0 for a
 * seq_len outside [1, L_max]).  rand_keys: DEVICE uint32 [B][Hkv][L_max].
 * Requires n_sink >= 0, n_recent >= 0, budget >= max(1, n_sink + n_recent). */
art_status art_evict_random_select(const art_shape* shape, const int32_t* seq_lens, const uint32_t* rand_keys,
                                   int32_t n_sink, int32_t n_recent, int32_t budget, int32_t* kept,
                                   int32_t* kept_lens, void* stream);

/* Pack rows: dst[b][h][i] = src[b][h][kept[b][h][i]] for the [B][Hkv][L_max][d]
 * cache `src` of the given format into dst [B][Hkv][budget][d]; q8 also packs its
 * scales (src_scale [B][Hkv][L_max][d/32] -> dst_scale [B][Hkv][budget][d/32];
 * pass NULL for both otherwise).  Rows whose index is -1 (or outside [0, L_max))
 * are written as zeros.  Call once for K and once for V. */
art_status art_evict_compact(const art_shape* shape, art_kv_format format, const void* src,
                             const uint16_t* src_scale, const int32_t* kept, int32_t budget, void* dst,
                             uint16_t* dst_scale, void* stream);

/* Synchronise `stream`, read the sticky status word of ws, clear it, and
 * return ART_OK, ART_ERR_SEQLEN, ART_ERR_TIMEOUT, ART_ERR_ORDER or ART_ERR_PAGE
 * (ART_ERR_CUDA if the synchronisation or copy failed). */
art_status art_read_device_status(void* ws, void* stream);

/* Base name of the CUDA kernel a call with this shape would launch for its
 * main pass: "art_decode_tc_kernel" (tcgen05 tensor-core path: bf16, d = 128,
 * tile 64 or 128, Hq/Hkv <= 8, full or ART) or "art_decode_kernel" (CUDA-core
 * path, everything else); NULL for an invalid or unsupported shape.  kv_q8 != 0
 * asks about art_decode_attn_q8_skipv (dtype is then ignored); with_art != 0
 * about the ART variant.  q8 without ART names the second of the two passes
 * that run when the workspace holds art_q8_workspace_bytes: "q8_pv_mma_kernel"
 * (tensor cores; d = 128, tile >= 32, 3 or 4 heads per kv head) or "q8_pv_kernel";
 * q8 with ART on such a shape names "q8_pv_mma_kernel" too (the passes that run
 * with that workspace: scores, probe pass, rule, limited pass, combine).  A query only: no CUDA call, nothing enqueued.  The
 * pages have no counterpart; it names the kernel for profiling and reports.
 * With num_splits > 1 a second, small kernel (art_combine_kernel) follows. */
const char* art_kernel_name(const art_shape* shape, art_dtype dtype, int32_t kv_q8, int32_t with_art);

/* Static, human-readable name of a status code. */
const char* art_status_string(art_status status);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* ART_DECODE_H */
