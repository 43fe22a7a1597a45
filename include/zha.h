/*
 * zha.h - C ABI of libzha: B200 (sm_100a) tree build and tree-routed sparse decode for
 * Zyphra Hierarchical Attention (ZHA).
 *
 * What the operations compute (pages cited by title and section):
 *  - Tree build: "Zyphra ZHA 稀疏注意力：8.2 万参数与 373 倍加速推算" (fluxbbs.com),
 *    section "树形索引是怎么搭的"; "Zyphra发布层级注意力ZHA：稀疏搜索实现亚二次复杂度"
 *    (wqu.guru), section "Building the tree".  Keys are cut into contiguous chunks of C
 *    tokens; for each of R reference queries q_r a chunk is summarised by the tangent
 *    plane of its log attention mass at q_r: lse_r = log sum_t exp(s q_r.k_t) and slope
 *    m_r = softmax-weighted mean of the keys (s = 1/sqrt(d)); b_r = lse_r - s q_r.m_r.
 *    Summaries are merged upward one level at a time: a level-l node covers C^l tokens;
 *    this library merges the C children's (lse_r, m_r) with the online-softmax combine,
 *    which equals the summary of the C^l raw tokens.
 *  - Routing: fluxbbs section "树形索引是怎么搭的"; wqu.guru section "How does top-p
 *    routing pick tokens?".  Per query head, the complete
 *    top-level nodes are scored by max_r (s q.m_r + b_r); at each level the smallest
 *    (score desc, index asc) prefix of the candidates whose softmax mass over the
 *    candidates reaches p is kept, and only the kept nodes' children are scored next.
 *  - Sparse attention: fluxbbs section "树形索引是怎么搭的" (exact attention over the raw
 *    rows routing keeps), wqu.guru section "How does top-p routing pick tokens?" (token 0
 *    attended as a sink every time).  Exact softmax attention
 *    over token 0, the tokens of the kept level-1 chunks and the tail of tokens after the
 *    last complete top node.
 *
 * Conventions
 *  - Every device pointer is a CUDA device address on the current device; the caller
 *    owns K, V, Q, q_ref and output buffers.  The library owns tree storage and decode
 *    workspace (allocated at create time, freed at destroy time).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is enqueued
 *    asynchronously on it; functions do not synchronise unless stated.
 *  - bf16 means IEEE bfloat16 bit patterns (uint16); f32 outputs are IEEE binary32.
 *  - Device pointers must be 16-byte aligned.
 *  - Functions return a zha_status; on failure nothing was enqueued, and
 *    zha_last_error() returns a message for the calling thread.  No exception crosses
 *    the ABI.  Objects are not thread-safe; use one thread per object at a time.
 *  - Conditions only a kernel can see (the device status word, bits listed at
 *    zha_decoder_stats) are reported by the routing and attention calls themselves: see
 *    zha_decoder_set_sync.  No kernel traps.
 */
#ifndef ZHA_H
#define ZHA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZHA_MAX_LEVELS 16

typedef enum zha_status {
    ZHA_OK = 0,
    ZHA_ERR_ARG = 1,       /* null/misaligned pointer, bad size or geometry */
    ZHA_ERR_CAPACITY = 2,  /* a size exceeds what the object was created for */
    ZHA_ERR_CUDA = 3,      /* a CUDA runtime call failed (message in zha_last_error) */
    ZHA_ERR_STATE = 4,     /* call out of order (append before build, n_old mismatch, ...) */
    ZHA_ERR_DEVICE = 5     /* a kernel flagged an internal failure in the device status word */
} zha_status;

/* How a node record stores its R slopes m_r (b, lse and every computation stay f32).
 * The pages test a router with reduced-precision summaries next to the full one (wqu.guru,
 * summary bullets: an FP4 router variant); this library offers three formats:
 *   ZHA_SUMMARY_F16X2  m as two fp16 planes hi + lo (m = hi + lo within 2^-22 |m| + 2^-25):
 *                      float32-grade summaries, 4 bytes per value.  Keys must stay below
 *                      65504 in magnitude.  The default.
 *   ZHA_SUMMARY_BF16   m as one bf16 plane (relative rounding 2^-9): half the bytes every
 *                      scored node costs, one tensor-core pass per node; routing decisions
 *                      follow the rounded slopes, so kept sets differ from the float32-grade
 *                      router's where estimates are close.
 *   ZHA_SUMMARY_FP4    m as MXFP4 (OCP Microscaling Formats v1.0): 4-bit E2M1 codes with one
 *                      power-of-two E8M0 scale per 32 dims, 2^(floor(log2 max|block|) - 2);
 *                      values rounded to nearest (ties to even), above 6 x scale saturated.
 *                      About 1/7 of the two-plane bytes per scored node (1,152 B at R = 16,
 *                      d = 128).  Level-1 slopes are the MXFP4 rounding of the exact slopes;
 *                      merges read the stored (decoded) children, so the levels above carry
 *                      the rounding of the levels below.  Scored on the CUDA cores
 *                      (ZHA_KERNELS_TENSOR is refused); built by the streaming kernels. */
typedef enum zha_summary_format {
    ZHA_SUMMARY_F16X2 = 0,
    ZHA_SUMMARY_BF16 = 1,
    ZHA_SUMMARY_FP4 = 2
} zha_summary_format;

/* Tree geometry and the shape of the KV cache it indexes. */
typedef struct zha_geometry {
    int32_t C;            /* children per node = tokens per level-1 chunk, 2..1024 */
    int32_t L;            /* levels, 1..ZHA_MAX_LEVELS; a top node covers C^L tokens */
    int32_t R;            /* reference queries per KV head: 1, 2, 4, 8, 16 or 32 */
    int32_t d;            /* head dimension: 64 or 128 */
    int32_t n_q_heads;    /* query heads Hq (multiple of n_kv_heads) */
    int32_t n_kv_heads;   /* KV heads Hkv; query head h reads KV head h*Hkv/Hq */
    int64_t capacity;     /* rows per KV head of the K/V buffers (max tokens) */
    int32_t format;       /* zha_summary_format of the node records */
} zha_geometry;

typedef struct zha_tree zha_tree;        /* per-sequence summary tree (device memory) */
typedef struct zha_decoder zha_decoder;  /* routing + attention workspace for a batch of trees */

/* Message for the last failed call on this thread ("" if none).  Never NULL. */
const char* zha_last_error(void);

/* ------------------------------------------------------------------ tree */

/* Allocates the tree for `g` (levels 1..L at capacity: node records of the slopes in
 * g->format plus b [R] f32, rounded up to 8 floats, plus lse [R] f32 per node, plus q_ref).
 * *out receives the handle.  ZHA_ERR_ARG on invalid geometry, ZHA_ERR_CUDA on allocation
 * failure. */
zha_status zha_tree_create(const zha_geometry* g, zha_tree** out);

/* Frees the tree (synchronises the device first).  NULL is accepted. */
zha_status zha_tree_destroy(zha_tree* t);

/* Geometry, current token count, complete nodes per level (level_nodes[l-1] = n_tokens
 * / C^l, array of L entries, nullable) and device bytes held (nullable). Host only. */
zha_status zha_tree_info(const zha_tree* t, zha_geometry* g, int64_t* n_tokens,
                         int64_t* level_nodes, int64_t* device_bytes);

/* Builds every complete node of levels 1..L over the first n_tokens rows of K.
 *   K      bf16 [n_kv_heads][capacity][d] (device), row t of head g at (g*capacity+t)*d
 *   q_ref  bf16 [n_kv_heads][R][d] (device), copied into the tree (used by append too)
 * 0 <= n_tokens <= capacity, else ZHA_ERR_CAPACITY. */
zha_status zha_build_tree(zha_tree* t, const void* K, int64_t n_tokens, const void* q_ref,
                          void* stream);

/* Grows the tree by n_new tokens whose keys are already in K rows [n_old, n_old+n_new):
 * summarises the chunks these tokens complete and merges every ancestor that becomes
 * complete.  n_old must equal the tree's token count (ZHA_ERR_STATE otherwise, also
 * before the first build); n_old + n_new <= capacity (ZHA_ERR_CAPACITY). */
zha_status zha_append(zha_tree* t, const void* K, int64_t n_old, int64_t n_new, void* stream);

/* Copies level `level` (1..L) summaries of all KV heads into device buffers:
 *   m [n_kv_heads][n_l][R][d], lse [n_kv_heads][n_l][R], b [n_kv_heads][n_l][R]  (f32)
 * with n_l = level_nodes[level-1].  Any pointer may be NULL to skip that array. */
zha_status zha_tree_export(const zha_tree* t, int32_t level, float* m, float* lse, float* b,
                           void* stream);

/* ------------------------------------------------------------------ decode */

/* Creates a decoder for a batch of n_seq trees (same d, Hq, Hkv and summary format; C, L,
 * R may differ per tree) and up to max_queries query tokens per sequence per call.
 * Workspace is sized from the trees' capacities; trees must outlive the decoder. */
zha_status zha_decoder_create(const zha_tree* const* trees, int32_t n_seq, int32_t max_queries,
                              zha_decoder** out);
zha_status zha_decoder_destroy(zha_decoder* dec);

/* Reporting of the device status word by zha_route, zha_sparse_attn, zha_dense_attn and
 * zha_decode (the word: bits listed at zha_decoder_stats; zha_route and zha_dense_attn
 * clear it, zha_sparse_attn adds to what the last zha_route set).  Each of these calls
 * ends by copying the word to pinned host memory behind its kernels.
 *   on = 0 (default, asynchronous): the call returns as soon as its work is enqueued.  The
 *          next of these calls on the decoder, if it starts after the earlier call's work
 *          has completed on the GPU, returns ZHA_ERR_DEVICE when that word was not 0 (the
 *          bits in zha_last_error) and enqueues nothing; an earlier call still running is
 *          reported by a later call or by zha_decoder_stats, which synchronises.  Each
 *          report is made once.
 *   on = 1 (synchronous): each call waits for its own work and returns ZHA_ERR_DEVICE
 *          when the word is not 0 at its end (outputs are then not valid).
 * Host-side failures are returned at once in both modes. */
zha_status zha_decoder_set_sync(zha_decoder* dec, int32_t on);

/* Routing for n_q query tokens per sequence.
 *   Q  bf16 [n_seq][n_q][Hq][d] (device).
 *   p  top-p mass, 0 < p <= 1 (p >= 1 keeps every node).
 * Lane x = (s*n_q + i)*Hq + h.  Kept sets of every level stay in the decoder (see
 * zha_decoder_export_kept).  Uses each tree's current token count. */
zha_status zha_route(zha_decoder* dec, const void* Q, int32_t n_q, float p, void* stream);

/* Exact attention of the routed lanes over token 0, the kept level-1 chunks and the tail.
 *   K, V  arrays of n_seq device pointers, bf16 [n_kv_heads][capacity][d] each
 *   Q     the same buffer given to zha_route
 *   out   f32 [n_seq][n_q][Hq][d] (device). */
zha_status zha_sparse_attn(zha_decoder* dec, const void* const* K, const void* const* V,
                           const void* Q, int32_t n_q, float* out, void* stream);

/* Which kernels a decoder uses (both choices give the same result up to float32
 * rounding).  ZHA_KERNELS_AUTO scores on the tensor cores (tcgen05, records fed by TMA)
 * at every lane count when every tree has R = 16 and fp16 or bf16 records (at one query
 * token the node scan then runs at the HBM rate), on the CUDA cores otherwise (MXFP4
 * records, R != 16), and attends on the tensor cores at every lane count; SIMT and TENSOR
 * force one kind (SIMT with at most 16 lanes per group, R = 16 and d = 128 takes the
 * few-lane CUDA-core scorer).
 *   score  plane estimates: CUDA-core fp32 FMA, or tcgen05 kind::f16 (ZHA_ERR_ARG for
 *          TENSOR unless every tree has R = 16).  With ZHA_SUMMARY_F16X2 records Q is
 *          taken in fp16 and each summary in two passes (hi, lo); the tensor path then
 *          needs every entry of Q and of the cache's keys below 65504 in magnitude (the
 *          fp16 range), else it sets bit 8 of the device status word (see
 *          zha_decoder_stats) and its plane estimates are not valid - select SIMT for such
 *          data.  With ZHA_SUMMARY_BF16 records Q stays bf16 and one pass is made.
 *   attn   exact attention: CUDA-core split-KV, or tcgen05 kind::f16 (S = Q K^T exact
 *          products, P split into bf16 hi + lo for P V) */
typedef enum zha_kernels { ZHA_KERNELS_AUTO = 0, ZHA_KERNELS_SIMT = 1, ZHA_KERNELS_TENSOR = 2 } zha_kernels;
zha_status zha_decoder_set_kernels(zha_decoder* dec, int32_t score, int32_t attn);

/* Exact attention over a routed token set that allocates no device memory.  The pages
 * have no counterpart: this is a service for callers that cannot allocate where they
 * attend (a process whose device memory is owned by someone else's allocator, or a
 * latency-critical loop that must not pay for an allocation and the synchronisation it
 * may imply).  It computes what zha_sparse_attn computes for one sequence, from the
 * caller's buffers alone:
 *   K, V   bf16 [Hkv][ld][d] (device); rows [0, n_tokens) are the cache
 *   C, L   the tree geometry (chunk size; the tail starts at (n_tokens / C^L) C^L)
 *   Q      bf16 [n_q][Hq][d] (device)
 *   kept1  uint32 [n_q*Hq][words] (device): level-1 kept bitmaps, lane x = i*Hq + h,
 *          e.g. from zha_decoder_export_kept(dec, 1, ...); words >= ceil(n_tokens/C/32).
 *          Only bits of chunks under complete top nodes count (chunk j < T C^L / C with
 *          T = n_tokens / C^L); bits at or after the tail's first chunk, and bits past
 *          n_tokens / C, are ignored (the tail is attended whole in any case)
 *   out    f32 [n_q][Hq][d] (device)
 * Working memory comes from one 16 MiB array in the library's device image, reserved on
 * every device that loads the library until the process exits; a call needing more
 * returns ZHA_ERR_CAPACITY with the byte count in zha_last_error() (about 11 MB for one
 * query token of 16 heads over 1M tokens at C = 4).  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress) with that device current; make
 * that first call before any stream capture.  All calls share the array and leave their
 * contents in it; each call clears what must start at zero, so back-to-back calls on one
 * stream are independent, but calls that can overlap on the GPU (different streams or
 * threads, same device) race on the array.  No cudaMalloc/cudaFree or allocating
 * library routine is called.  Each call waits for its own work on `stream` to finish and
 * reads the array's status word back: ZHA_ERR_DEVICE if a kernel set it (none is expected
 * to on this path). */
zha_status zha_sparse_attn_static(const void* K, const void* V, int64_t ld, int64_t n_tokens,
                                  int32_t C, int32_t L, int32_t Hq, int32_t Hkv, int32_t d,
                                  const void* Q, int32_t n_q, const uint32_t* kept1, int64_t words,
                                  float* out, void* stream);

/* Dense exact attention: every query lane over all n_tokens tokens of its sequence,
 *   o = sum_t softmax_t(s q.k_t) v_t,  t in [0, N),  s = 1/sqrt(d),
 * with no routing.  The pages measure the routed decode against dense attention over the
 * whole cache (the speedup of their figures); this is that comparison's dense side on the
 * same kernels: the split-KV attention (tcgen05 or CUDA cores, as zha_decoder_set_kernels
 * selects) with every token a tail token of every lane, then the split combine.  K, V, Q
 * and out as for zha_sparse_attn; the decoder's trees give only each sequence's token
 * count and chunk size (the split granularity) and must be built.  Needs no zha_route and
 * leaves the last route's kept sets as they were (a later zha_sparse_attn still attends
 * them).  ZHA_ERR_CAPACITY if n_q exceeds the decoder's max_queries. */
zha_status zha_dense_attn(zha_decoder* dec, const void* const* K, const void* const* V,
                          const void* Q, int32_t n_q, float* out, void* stream);

/* zha_route followed by zha_sparse_attn. */
zha_status zha_decode(zha_decoder* dec, const void* const* K, const void* const* V,
                      const void* Q, int32_t n_q, float p, float* out, void* stream);

/* Kept sets of the last zha_route at `level` (1..max L of the batch), as bitmaps:
 *   bits   uint32 [n_lanes][words] (device), bit j of lane x set iff node j kept;
 *          words = zha_decoder_words(dec, level); lanes whose tree has fewer levels
 *          get all-zero rows
 *   counts int32 [n_lanes] (device, nullable): kept nodes per lane. */
zha_status zha_decoder_export_kept(const zha_decoder* dec, int32_t level, uint32_t* bits,
                                   int32_t* counts, void* stream);
int64_t zha_decoder_words(const zha_decoder* dec, int32_t level);

/* Work counters of the last zha_route / zha_sparse_attn (synchronises `stream`):
 * nodes scored per level as the union over each (sequence, KV head) group of lanes and
 * as the per-lane sum, attended tokens (union per group and per-lane sum), and the
 * device status word (0 = ok; bit 1: the top-p select ran out of bisection steps,
 * bit 2: a union list reached its capacity, bit 4: a tensor-core wait gave up after 2 s,
 * bit 8: an input outside the fp16 range reached the tensor-core scorer, bit 16: a
 * sharded cut's boundary bin held more keys than the ranks can exchange).
 * Returns ZHA_ERR_DEVICE when the status word is not 0. */
typedef struct zha_decode_stats {
    int64_t union_nodes[ZHA_MAX_LEVELS];      /* index l-1 */
    int64_t lane_nodes[ZHA_MAX_LEVELS];
    int64_t union_tokens;
    int64_t lane_tokens;
    int64_t node_bytes;                       /* bytes read per scored node (m planes and b) */
    int32_t status;
} zha_decode_stats;
zha_status zha_decoder_stats(const zha_decoder* dec, zha_decode_stats* out, void* stream);


/* ------------------------------------------------------------------ sharded sequence */

/* One sequence whose tokens are split over `world` ranks (one GPU each, one process per
 * GPU), for contexts whose KV cache and tree do not fit one GPU: the tree is stored on top
 * of the whole raw cache, so it saves bandwidth, not capacity (ic.work, section
 * "四百倍加速只是纸面推演，局部改装与位置编码暗藏边界", bullet "风险"), while the pages aim the
 * method at contexts of hundreds of millions of tokens (fluxbbs.com, section "换架构与后续展望").
 *
 * Layout: rank r holds tokens [token_offset_r, token_offset_r + n_r) of the sequence in its
 * own K, V (same layout as zha_build_tree, row 0 = the shard's first token) and its own
 * tree built over those rows; token_offset_0 = 0, the ranges are consecutive in rank order,
 * every token_offset is a multiple of C^L, and every rank but the last holds a multiple of
 * C^L tokens (the sequence's tail lives on the last rank).  The sequence's level-1 nodes
 * must number at most 2^24 (the fixed-point masses of one level then sum below 2^63).
 *
 * Result: the same routing and attention as one tree over the whole sequence.  Every level's
 * top-p cut is taken over the union of all ranks' frontiers: each rank sums the same exact
 * fixed-point mass histogram, and the boundary bin is ordered by (score desc, GLOBAL node
 * index asc), so the kept nodes in each rank's range are exactly the single-tree kept nodes
 * there; attention runs per rank over its kept chunks (token 0 of the sequence, the sink,
 * on rank 0; the tail on the last rank) and the ranks' results are merged by their
 * log-sum-exp.
 *
 * Protocol (every rank makes the same calls and collectives in the same order; `lanes` =
 * n_q * n_q_heads):
 *   zha_shard_begin
 *   for level = L down to 1:
 *     zha_shard_score   then  all-reduce MAX ex.lane_max (int32), SUM ex.lane_cnt (int32)
 *     zha_shard_hist    then  all-reduce SUM ex.hist (64-bit integers)
 *     zha_shard_cut     then  all-gather ex.keys -> ex.keys_all, ex.nkeys -> ex.nkeys_all
 *     zha_shard_finish
 *   zha_shard_attend    then  all-gather ex.out -> ex.out_all, ex.lse -> ex.lse_all
 *   zha_shard_combine
 * A call out of this order returns ZHA_ERR_STATE and enqueues nothing.  The exchange
 * buffers are device memory owned by the caller (all 16-byte aligned); all-gathers are
 * rank-major ([world][...] with rank r's block at r). */
#define ZHA_SHARD_BINS 2048
#define ZHA_SHARD_KEYS 2048
typedef struct zha_shard_exchange {
    int32_t* lane_max;          /* [lanes] frontier maximum score, as ordered int32 (MAX over ranks) */
    int32_t* lane_cnt;          /* [lanes] frontier size (SUM over ranks) */
    uint64_t* hist;             /* [lanes][ZHA_SHARD_BINS] fixed-point bin masses (SUM over ranks) */
    uint64_t* keys;             /* [lanes][ZHA_SHARD_KEYS] this rank's boundary-bin keys */
    int32_t* nkeys;             /* [lanes] their number (may exceed ZHA_SHARD_KEYS: reported) */
    const uint64_t* keys_all;   /* [world][lanes][ZHA_SHARD_KEYS] gathered keys */
    const int32_t* nkeys_all;   /* [world][lanes] */
    float* out;                 /* [lanes][d] this rank's attention output (normalised) */
    float* lse;                 /* [lanes] its log-sum-exp of scaled scores (-inf: no token) */
    const float* out_all;       /* [world][lanes][d] */
    const float* lse_all;       /* [world][lanes] */
} zha_shard_exchange;

/* A decoder for this rank's shard: tree = the shard's tree; rank in [0, world);
 * token_offset = global index of the shard's first token (0 exactly for rank 0, else a
 * positive multiple of C^L).  Destroy with zha_decoder_destroy.  The routing calls of a
 * plain decoder (zha_route, zha_decode, ...) are refused on it (ZHA_ERR_STATE). */
zha_status zha_shard_decoder_create(const zha_tree* tree, int32_t max_queries, int32_t rank, int32_t world,
                                    int64_t token_offset, zha_decoder** out);
/* Q bf16 [n_q][n_q_heads][d] (device; kept until zha_shard_combine), p as in zha_route. */
zha_status zha_shard_begin(zha_decoder* dec, const void* Q, int32_t n_q, float p, void* stream);
zha_status zha_shard_score(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream);
zha_status zha_shard_hist(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream);
zha_status zha_shard_cut(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream);
/* The last step of a level.  A lane whose boundary bin held more than ZHA_SHARD_KEYS keys on
 * one rank, or more than 4,096 over all ranks, cannot be finished: bit 16 of the device
 * status word is set (reported by the level-1 finish and by zha_shard_combine, see
 * zha_decoder_set_sync). */
zha_status zha_shard_finish(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream);
/* K, V: this shard's rows (as zha_build_tree). */
zha_status zha_shard_attend(zha_decoder* dec, const void* K, const void* V, const zha_shard_exchange* ex,
                            void* stream);
/* out f32 [n_q][n_q_heads][d] (device): the sequence's attention output. */
zha_status zha_shard_combine(zha_decoder* dec, const zha_shard_exchange* ex, float* out, void* stream);


/* ------------------------------------------------------------------ profile */

/* Device-time profile of this library's own kernels (off by default; not part of the
 * method).  While enabled, every kernel launch is bracketed by two CUDA events recorded
 * on its launch stream (so launches must not be under stream capture).
 * zha_profile_read synchronises the device, sums the recorded intervals per kernel and
 * returns the number of distinct kernels seen; at most max_kernels entries are written:
 *   names     char [max_kernels][name_len] (host), NUL-terminated kernel names
 *   launches  int64 [max_kernels] (host);  total_ms  double [max_kernels] (host).
 * Any output pointer may be NULL.  zha_profile_reset drops the recorded intervals. */
zha_status zha_profile_enable(int32_t on);
int32_t zha_profile_read(char* names, int32_t name_len, int64_t* launches, double* total_ms,
                         int32_t max_kernels);
zha_status zha_profile_reset(void);

#ifdef __cplusplus
}
#endif
#endif /* ZHA_H */
