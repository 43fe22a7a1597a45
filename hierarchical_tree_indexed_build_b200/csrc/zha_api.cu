// zha_api.cu - the C ABI declared in include/zha.h: object lifetime, argument checks and
// the launch sequences of tree build, append, routing and sparse attention.
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "zha_common.cuh"
#include "zha_launch.h"

using namespace zha;

namespace {

thread_local std::string g_err;

zha_status fail(zha_status s, const std::string& msg) {
    g_err = msg;
    return s;
}

#define ZHA_CUDA(expr)                                                                     \
    do {                                                                                   \
        cudaError_t e_ = (expr);                                                           \
        if (e_ != cudaSuccess) return fail(ZHA_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ipow(int64_t c, int l) {
    int64_t r = 1;
    for (int i = 0; i < l; ++i) r *= c;
    return r;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

float score_scale(int d) { return (float)(1.0 / sqrt((double)d)); }

// TMA maps of one level (fp16 planes viewed as (dim, plane r, hi/lo, node over all KV
// heads), 128-byte swizzle = the MMA operand layout; b viewed as (r, node)):
//   maps[0] planes, boxes of 64 dims x R planes x 1 node
//   maps[1] planes, boxes of 64 dims x R planes x 4 nodes
//   maps[2] b, boxes of R values x 4 nodes
bool encode_level_maps(CUtensorMap* maps, const float* rec, int d, int R, int64_t nodes, int ns, int fmt) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    // planes viewed as (dim, slope r, plane, node): two fp16 planes, or one bf16 plane
    const cuuint64_t planes = fmt == kFmtBf16 ? 1 : 2;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)R, planes, (cuuint64_t)nodes};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)R * d * 2, (cuuint64_t)ns * 4};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = fmt == kFmtBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    for (int k = 0; k < 2; ++k) {
        const cuuint32_t box[4] = {64, (cuuint32_t)R, 1, k == 0 ? 1u : 4u};
        if (encode(&maps[k], dt, 4, const_cast<float*>(rec), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    const cuuint64_t bdims[2] = {(cuuint64_t)R, (cuuint64_t)nodes};
    const cuuint64_t bstrides[1] = {(cuuint64_t)ns * 4};
    const cuuint32_t bbox[2] = {(cuuint32_t)R, 4};
    const cuuint32_t bestr[2] = {1, 1};
    return encode(&maps[2], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(rec) + b_offset(R, d, fmt), bdims,
                  bstrides, bbox, bestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

struct zha_tree {
    zha_geometry g;
    int32_t ns;
    int64_t n_tokens;
    bool built;
    int64_t cap[kMaxL + 1];
    float* rec[kMaxL + 1];
    float* lse[kMaxL + 1];
    __nv_bfloat16* qref;
    int32_t* rflag;          // device word: a summary left the fp16 range
    void* block;
    size_t bytes;
    int device;
};

struct zha_decoder {
    std::vector<const zha_tree*> trees;
    int32_t n_seq, max_q, Hq, Hkv, d, G, Lmax;
    int64_t lanes_cap, groups_cap;
    int64_t part_slots;   // attention partial records: lanes x splits of one call
    Work w;
    SeqDev* seq_dev;
    std::vector<SeqDev> seq_host;
    void* block;
    size_t bytes;
    int32_t last_n_q;
    bool routed;
    int32_t score_path;
    int32_t attn_path;
    int32_t all_r16;
    // Device status word as the host sees it: every routing / attention call ends by copying
    // the word into pinned host memory and recording `status_ev` after the copy.
    int32_t* status_host;
    cudaEvent_t status_ev;
    bool status_pending;     // a copy was enqueued and not yet looked at
    int32_t sync;            // calls wait for their own work and report its status
    // Sequence-sharded decode (zha_shard_*); sh_world = 0 on a plain decoder.
    int32_t sh_rank = 0, sh_world = 0;
    int64_t sh_tok0 = 0;             // global index of the shard's first token
    unsigned long long* sh_need = nullptr;   // [lanes_cap] (workspace)
    const void* sh_Q = nullptr;
    int32_t sh_nq = 0;
    float sh_p = 1.0f;
    int32_t sh_level = 0;            // level of the next protocol step (0: attention)
    int32_t sh_step = -1;            // next step: 0 score, 1 hist, 2 cut, 3 finish, 4 attend, 5 combine; -1 none
};

extern "C" const char* zha_last_error(void) { return g_err.c_str(); }

zha_status zha::set_last_error(zha_status s, const char* msg) { return fail(s, msg); }

// ------------------------------------------------------------------------------ tree

static zha_status check_geometry(const zha_geometry* g) {
    if (!g) return fail(ZHA_ERR_ARG, "geometry is NULL");
    if (g->C < 2 || g->C > 1024) return fail(ZHA_ERR_ARG, "C must be in [2, 1024]");
    if (g->L < 1 || g->L > kMaxL) return fail(ZHA_ERR_ARG, "L must be in [1, 16]");
    if (!(g->R == 1 || g->R == 2 || g->R == 4 || g->R == 8 || g->R == 16 || g->R == 32))
        return fail(ZHA_ERR_ARG, "R must be 1, 2, 4, 8, 16 or 32");
    if (g->d != 64 && g->d != 128) return fail(ZHA_ERR_ARG, "d must be 64 or 128");
    if (g->n_kv_heads < 1 || g->n_q_heads < g->n_kv_heads || g->n_q_heads % g->n_kv_heads)
        return fail(ZHA_ERR_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
    if (g->capacity < 1 || g->capacity > (int64_t(1) << 31) - 1)
        return fail(ZHA_ERR_ARG, "capacity must be in [1, 2^31)");
    if (g->capacity / g->C > (int64_t(1) << 24))
        return fail(ZHA_ERR_ARG, "capacity / C must be <= 2^24 level-1 nodes");
    double top = pow((double)g->C, (double)g->L);
    if (top > 4.0e15) return fail(ZHA_ERR_ARG, "C^L too large");
    if (g->format != ZHA_SUMMARY_F16X2 && g->format != ZHA_SUMMARY_BF16 && g->format != ZHA_SUMMARY_FP4)
        return fail(ZHA_ERR_ARG, "format must be ZHA_SUMMARY_F16X2, ZHA_SUMMARY_BF16 or ZHA_SUMMARY_FP4");
    return ZHA_OK;
}

extern "C" zha_status zha_tree_create(const zha_geometry* g, zha_tree** out) {
    zha_status st = check_geometry(g);
    if (st != ZHA_OK) return st;
    if (!out) return fail(ZHA_ERR_ARG, "out is NULL");
    zha_tree* t = new zha_tree();
    memset(t, 0, sizeof(*t));
    t->g = *g;
    t->ns = record_stride(g->R, g->d, g->format);
    size_t off = 0;
    size_t rec_off[kMaxL + 1] = {0}, lse_off[kMaxL + 1] = {0};
    for (int l = 1; l <= g->L; ++l) {
        const int64_t span = ipow(g->C, l);
        t->cap[l] = g->capacity / span;
        rec_off[l] = off;
        off += up256((size_t)g->n_kv_heads * t->cap[l] * t->ns * sizeof(float));
        lse_off[l] = off;
        off += up256((size_t)g->n_kv_heads * t->cap[l] * g->R * sizeof(float));
    }
    const size_t qref_off = off;
    off += up256((size_t)g->n_kv_heads * g->R * g->d * 2);
    const size_t rflag_off = off;
    off += up256(4);
    cudaGetDevice(&t->device);
    cudaError_t e = cudaMalloc(&t->block, off);
    if (e != cudaSuccess) {
        delete t;
        return fail(ZHA_ERR_CUDA, std::string("cudaMalloc(tree): ") + cudaGetErrorString(e));
    }
    t->bytes = off;
    char* base = static_cast<char*>(t->block);
    for (int l = 1; l <= g->L; ++l) {
        t->rec[l] = reinterpret_cast<float*>(base + rec_off[l]);
        t->lse[l] = reinterpret_cast<float*>(base + lse_off[l]);
    }
    t->qref = reinterpret_cast<__nv_bfloat16*>(base + qref_off);
    t->rflag = reinterpret_cast<int32_t*>(base + rflag_off);
    cudaMemset(t->rflag, 0, 4);
    *out = t;
    return ZHA_OK;
}

extern "C" zha_status zha_tree_destroy(zha_tree* t) {
    if (!t) return ZHA_OK;
    cudaDeviceSynchronize();
    cudaFree(t->block);
    delete t;
    return ZHA_OK;
}

extern "C" zha_status zha_tree_info(const zha_tree* t, zha_geometry* g, int64_t* n_tokens,
                                    int64_t* level_nodes, int64_t* device_bytes) {
    if (!t) return fail(ZHA_ERR_ARG, "tree is NULL");
    if (g) *g = t->g;
    if (n_tokens) *n_tokens = t->n_tokens;
    if (level_nodes)
        for (int l = 1; l <= t->g.L; ++l) level_nodes[l - 1] = t->n_tokens / ipow(t->g.C, l);
    if (device_bytes) *device_bytes = (int64_t)t->bytes;
    return ZHA_OK;
}

// Summaries of every node completed by growing the token count from n_old to n_new.
static zha_status run_levels(zha_tree* t, const void* K, int64_t n_old, int64_t n_new, cudaStream_t st) {
    const zha_geometry& g = t->g;
    const int C = g.C, L = g.L;
    BuildArgs ba;
    memset(&ba, 0, sizeof(ba));
    ba.K = static_cast<const __nv_bfloat16*>(K);
    ba.ld = g.capacity;
    ba.qref = t->qref;
    ba.rflag = t->rflag;
    ba.Hkv = g.n_kv_heads;
    ba.R = g.R;
    ba.C = C;
    ba.ns = t->ns;
    ba.fmt = g.format;
    ba.scale = score_scale(g.d);
    for (int l = 1; l <= L; ++l) {
        ba.rec[l] = t->rec[l];
        ba.lse[l] = t->lse[l];
        ba.cap[l] = t->cap[l];
    }
    auto merge = [&](int l, int64_t lo, int64_t hi) -> zha_status {
        if (hi <= lo) return ZHA_OK;
        MergeArgs ma;
        memset(&ma, 0, sizeof(ma));
        ma.qref = t->qref;
        ma.rflag = t->rflag;
        ma.Hkv = g.n_kv_heads;
        ma.R = g.R;
        ma.C = C;
        ma.ns = t->ns;
        ma.fmt = g.format;
        ma.p0 = lo;
        ma.np = hi - lo;
        ma.scale = score_scale(g.d);
        ma.child_rec = t->rec[l - 1];
        ma.child_lse = t->lse[l - 1];
        ma.child_cap = t->cap[l - 1];
        ma.rec = t->rec[l];
        ma.lse = t->lse[l];
        ma.cap = t->cap[l];
        ZHA_CUDA(launch_merge(ma, g.d, st));
        return ZHA_OK;
    };
    if (build_tc_supported(C, g.R, g.d, g.format)) {
        // levels 1..3 on the tensor cores, over whole 128-token tiles holding a new chunk (the
        // tile's other nodes are rewritten with the same bits); the levels above by merges
        const int k_emit = std::min(3, L);
        const int64_t lo = n_old / C, hi = n_new / C;
        if (hi > lo) {
            BuildTcArgs ta;
            memset(&ta, 0, sizeof(ta));
            ta.K = static_cast<const __nv_bfloat16*>(K);
            ta.ld = g.capacity;
            ta.n_tokens = n_new;
            ta.qref = t->qref;
            ta.rflag = t->rflag;
            ta.Hkv = g.n_kv_heads;
            ta.ns = t->ns;
            ta.k_emit = k_emit;
            ta.t0 = lo / 32;
            ta.t1 = (hi - 1) / 32 + 1;
            ta.n1 = n_new / C;
            ta.n2 = n_new / (C * C);
            ta.n3 = n_new / (C * C * C);
            ta.scale = score_scale(g.d);
            for (int l = 1; l <= k_emit; ++l) {
                ta.rec[l] = t->rec[l];
                ta.lse[l] = t->lse[l];
                ta.cap[l] = t->cap[l];
            }
            ZHA_CUDA(launch_build_tc(ta, g.d, st));
        }
        for (int l = k_emit + 1; l <= L; ++l) {
            const int64_t span = ipow(C, l);
            zha_status s2 = merge(l, n_old / span, n_new / span);
            if (s2 != ZHA_OK) return s2;
        }
        return ZHA_OK;
    }
    int first_merge = 2;
    int64_t lo1 = n_old / C;
    if (n_old == 0) {
        // Whole subtrees of up to 64 tokens are streamed by one worker each (more workers in
        // flight than with larger spans; the levels above come from merges).
        int k_emit = 1;
        while (k_emit < L && ipow(C, k_emit + 1) <= 64) ++k_emit;
        const int64_t n_emit = n_new / ipow(C, k_emit);
        ba.k_emit = k_emit;
        ba.u0 = 0;
        ba.nu = n_emit;
        ZHA_CUDA(launch_build_stream(ba, g.d, st));
        lo1 = n_emit * ipow(C, k_emit - 1);
        ba.k_emit = 1;
        ba.u0 = lo1;
        ba.nu = n_new / C - lo1;
        ZHA_CUDA(launch_build_stream(ba, g.d, st));
        for (int l = 2; l <= k_emit; ++l) {
            zha_status s2 = merge(l, n_emit * ipow(C, k_emit - l), n_new / ipow(C, l));
            if (s2 != ZHA_OK) return s2;
        }
        first_merge = k_emit + 1;
        for (int l = first_merge; l <= L; ++l) {
            zha_status s2 = merge(l, 0, n_new / ipow(C, l));
            if (s2 != ZHA_OK) return s2;
        }
        return ZHA_OK;
    }
    ba.k_emit = 1;
    ba.u0 = lo1;
    ba.nu = n_new / C - lo1;
    ZHA_CUDA(launch_build_stream(ba, g.d, st));
    for (int l = 2; l <= L; ++l) {
        const int64_t span = ipow(C, l);
        zha_status s2 = merge(l, n_old / span, n_new / span);
        if (s2 != ZHA_OK) return s2;
    }
    return ZHA_OK;
}

extern "C" zha_status zha_build_tree(zha_tree* t, const void* K, int64_t n_tokens, const void* q_ref,
                                     void* stream) {
    if (!t) return fail(ZHA_ERR_ARG, "tree is NULL");
    if (!K || !q_ref) return fail(ZHA_ERR_ARG, "K or q_ref is NULL");
    if (!aligned16(K) || !aligned16(q_ref)) return fail(ZHA_ERR_ARG, "K and q_ref must be 16-byte aligned");
    if (n_tokens < 0 || n_tokens > t->g.capacity)
        return fail(ZHA_ERR_CAPACITY, "n_tokens must be in [0, capacity]");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(cudaMemcpyAsync(t->qref, q_ref, (size_t)t->g.n_kv_heads * t->g.R * t->g.d * 2,
                             cudaMemcpyDeviceToDevice, st));
    ZHA_CUDA(cudaMemsetAsync(t->rflag, 0, 4, st));
    zha_status s = run_levels(t, K, 0, n_tokens, st);
    if (s != ZHA_OK) return s;
    t->n_tokens = n_tokens;
    t->built = true;
    return ZHA_OK;
}

extern "C" zha_status zha_append(zha_tree* t, const void* K, int64_t n_old, int64_t n_new, void* stream) {
    if (!t) return fail(ZHA_ERR_ARG, "tree is NULL");
    if (!t->built) return fail(ZHA_ERR_STATE, "append before zha_build_tree");
    if (!K || !aligned16(K)) return fail(ZHA_ERR_ARG, "K must be a 16-byte aligned device pointer");
    if (n_old != t->n_tokens) return fail(ZHA_ERR_STATE, "n_old differs from the tree's token count");
    if (n_new < 0) return fail(ZHA_ERR_ARG, "n_new must be >= 0");
    if (n_old + n_new > t->g.capacity) return fail(ZHA_ERR_CAPACITY, "n_old + n_new exceeds capacity");
    if (n_new == 0) return ZHA_OK;
    zha_status s = run_levels(t, K, n_old, n_old + n_new, static_cast<cudaStream_t>(stream));
    if (s != ZHA_OK) return s;
    t->n_tokens = n_old + n_new;
    return ZHA_OK;
}

extern "C" zha_status zha_tree_export(const zha_tree* t, int32_t level, float* m, float* lse, float* b,
                                      void* stream) {
    if (!t) return fail(ZHA_ERR_ARG, "tree is NULL");
    if (level < 1 || level > t->g.L) return fail(ZHA_ERR_ARG, "level out of range");
    const zha_geometry& g = t->g;
    const int64_t nl = t->n_tokens / ipow(g.C, level);
    if (nl == 0) return ZHA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m) ZHA_CUDA(launch_export_m(t->rec[level], t->cap[level], t->ns, g.n_kv_heads, g.R, g.d, g.format, nl, m, st));
    for (int h = 0; h < g.n_kv_heads; ++h) {
        const float* src = t->rec[level] + (int64_t)h * t->cap[level] * t->ns;
        if (b)
            ZHA_CUDA(cudaMemcpy2DAsync(b + (int64_t)h * nl * g.R, (size_t)g.R * 4, src + b_offset(g.R, g.d, g.format),
                                       (size_t)t->ns * 4, (size_t)g.R * 4, (size_t)nl,
                                       cudaMemcpyDeviceToDevice, st));
        if (lse)
            ZHA_CUDA(cudaMemcpyAsync(lse + (int64_t)h * nl * g.R, t->lse[level] + (int64_t)h * t->cap[level] * g.R,
                                     (size_t)nl * g.R * 4, cudaMemcpyDeviceToDevice, st));
    }
    return ZHA_OK;
}

// ------------------------------------------------------------------------------ decoder

extern "C" zha_status zha_decoder_create(const zha_tree* const* trees, int32_t n_seq, int32_t max_queries,
                                         zha_decoder** out) {
    if (!trees || n_seq < 1) return fail(ZHA_ERR_ARG, "need at least one tree");
    if (max_queries < 1) return fail(ZHA_ERR_ARG, "max_queries must be >= 1");
    if (!out) return fail(ZHA_ERR_ARG, "out is NULL");
    for (int s = 0; s < n_seq; ++s) {
        if (!trees[s]) return fail(ZHA_ERR_ARG, "a tree is NULL");
        const zha_geometry& a = trees[s]->g;
        const zha_geometry& b0 = trees[0]->g;
        if (a.d != b0.d || a.n_q_heads != b0.n_q_heads || a.n_kv_heads != b0.n_kv_heads || a.format != b0.format)
            return fail(ZHA_ERR_ARG, "trees of one decoder must share d, n_q_heads, n_kv_heads and format");
    }
    zha_decoder* dec = new zha_decoder();
    dec->trees.assign(trees, trees + n_seq);
    const zha_geometry& g0 = trees[0]->g;
    dec->n_seq = n_seq;
    dec->max_q = max_queries;
    dec->Hq = g0.n_q_heads;
    dec->Hkv = g0.n_kv_heads;
    dec->d = g0.d;
    dec->G = g0.n_q_heads / g0.n_kv_heads;
    dec->Lmax = 0;
    for (auto* t : dec->trees) dec->Lmax = t->g.L > dec->Lmax ? t->g.L : dec->Lmax;
    dec->lanes_cap = (int64_t)n_seq * max_queries * dec->Hq;
    dec->groups_cap = (int64_t)n_seq * dec->Hkv;
    dec->last_n_q = 0;
    dec->routed = false;
    dec->score_path = ZHA_KERNELS_AUTO;
    dec->attn_path = ZHA_KERNELS_AUTO;
    dec->all_r16 = 1;
    for (auto* t : dec->trees) dec->all_r16 &= (t->g.R == 16) ? 1 : 0;

    Work& w = dec->w;
    memset(&w, 0, sizeof(w));
    int64_t cap1 = 1, part_slots = 1;
    for (int l = 1; l <= dec->Lmax; ++l) {
        int64_t W = 1;
        for (auto* t : dec->trees)
            if (l <= t->g.L) W = std::max<int64_t>(W, (t->cap[l] + 31) / 32);
        w.W[l] = (W + 7) / 8 * 8;   // rows of whole 32-byte segments (vector reads of 256-node spans)
    }
    for (auto* t : dec->trees) {
        cap1 = std::max<int64_t>(cap1, t->cap[1]);
        const int64_t top = ipow(t->g.C, t->g.L);
        const int64_t nseg_max = 1 + t->cap[1] + (std::min<int64_t>(top, t->g.capacity) + t->g.C - 1) / t->g.C;
        // attention partials: the most lanes x splits any call can need.  The split size
        // depends on the lanes per group (decoder_split_tokens), so take the largest query
        // count of each split-size bucket (<= 16, <= 64, more lanes per group).
        for (int bk = 0; bk < 3; ++bk) {
            const int64_t gl_lim = bk == 0 ? 16 : (bk == 1 ? 64 : (int64_t)max_queries * dec->G);
            const int64_t nq = std::min<int64_t>(max_queries, gl_lim / dec->G);
            if (nq < 1) continue;
            const int64_t segs = std::max<int64_t>(1, decoder_split_tokens((int)(nq * dec->G)) / t->g.C);
            const int64_t lanes = (int64_t)n_seq * nq * dec->Hq;
            part_slots = std::max<int64_t>(part_slots, lanes * ((nseg_max + segs - 1) / segs));
        }
    }
    // union lists whose lane masks are transposed: parents of a scored level (level >= 2)
    // and the kept level-1 chunks attention gathers
    w.ms = cap1;
    w.mwords = (max_queries * dec->G + 255) / 256 * 8;
    w.lanes_cap = dec->lanes_cap;
    w.es = (cap1 + 127) / 128 * 128;   // score rows padded to whole 128-candidate blocks
    w.us = (cap1 + 7) / 8 * 8 + 8;   // union lists: room for 16-byte-rounded bulk reads past the end
    w.s_cap = 0;   // the partials' split stride, set per call
    dec->part_slots = part_slots;

    size_t off = 0;
    size_t kept_off[kMaxL + 2] = {0};
    for (int l = 1; l <= dec->Lmax; ++l) {
        kept_off[l] = off;
        off += up256((size_t)dec->lanes_cap * w.W[l] * 4);
    }
    const size_t kcount_off = off;
    off += up256((size_t)(kMaxL + 1) * dec->lanes_cap * 4);
    const size_t e_off = off;
    off += up256((size_t)dec->lanes_cap * w.es * 4);
    const size_t ulist_off = off;
    off += up256((size_t)dec->groups_cap * w.us * 4);
    const size_t ucount_off = off;
    off += up256((size_t)dec->groups_cap * 4);
    w.uw = w.W[1];
    const size_t uword_off = off;
    off += up256((size_t)dec->groups_cap * w.uw * 4);
    const size_t part_off = off;
    off += up256((size_t)part_slots * (dec->d + 4) * 4);
    const size_t memb_off = off;
    off += up256((size_t)dec->groups_cap * w.ms * w.mwords * 4);
    const size_t lmax_off = off;
    off += up256((size_t)(kMaxL + 1) * dec->lanes_cap * 4);
    const size_t lcnt_off = off;
    off += up256((size_t)(kMaxL + 1) * dec->lanes_cap * 4);
    const size_t tmap_off = off;
    off += up256((size_t)n_seq * (kMaxL + 1) * kMapsPerLevel * sizeof(CUtensorMap));
    const size_t ctr_off = off;
    off += up256((size_t)kCtrCount * 8);
    const size_t status_off = off;
    off += up256(4);
    const size_t seq_off = off;
    off += up256((size_t)n_seq * sizeof(SeqDev));
    const size_t need_off = off;
    off += up256((size_t)dec->lanes_cap * 8);
    cudaError_t e = cudaMalloc(&dec->block, off);
    if (e != cudaSuccess) {
        delete dec;
        return fail(ZHA_ERR_CUDA, std::string("cudaMalloc(decoder workspace): ") + cudaGetErrorString(e));
    }
    dec->bytes = off;
    char* base = static_cast<char*>(dec->block);
    for (int l = 1; l <= dec->Lmax; ++l) w.kept[l] = reinterpret_cast<uint32_t*>(base + kept_off[l]);
    w.kcount = reinterpret_cast<int32_t*>(base + kcount_off);
    w.e = reinterpret_cast<float*>(base + e_off);
    w.ulist = reinterpret_cast<int32_t*>(base + ulist_off);
    w.ucount = reinterpret_cast<int32_t*>(base + ucount_off);
    w.uword = reinterpret_cast<uint32_t*>(base + uword_off);
    w.part = reinterpret_cast<float*>(base + part_off);
    w.memb = reinterpret_cast<uint32_t*>(base + memb_off);
    w.lane_max = reinterpret_cast<uint32_t*>(base + lmax_off);
    w.lane_cnt = reinterpret_cast<int32_t*>(base + lcnt_off);
    w.ctr = reinterpret_cast<unsigned long long*>(base + ctr_off);
    w.status = reinterpret_cast<int32_t*>(base + status_off);
    dec->seq_dev = reinterpret_cast<SeqDev*>(base + seq_off);
    dec->sh_need = reinterpret_cast<unsigned long long*>(base + need_off);
    dec->seq_host.resize(n_seq);
    // TMA maps of the trees' fp16 (or bf16) planes, one per (sequence, level), for the tensor
    // scorer; MXFP4 records are scored on the CUDA cores only
    w.tmaps = nullptr;
    if (dec->all_r16 && g0.format != ZHA_SUMMARY_FP4) {
        std::vector<CUtensorMap> maps((size_t)n_seq * (kMaxL + 1) * kMapsPerLevel);
        memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
        bool ok = true;
        for (int s = 0; s < n_seq && ok; ++s) {
            const zha_tree* t = dec->trees[s];
            for (int l = 1; l <= t->g.L && ok; ++l)
                ok = encode_level_maps(&maps[((size_t)s * (kMaxL + 1) + l) * kMapsPerLevel], t->rec[l], t->g.d, t->g.R,
                                       (int64_t)t->g.n_kv_heads * t->cap[l], t->ns, t->g.format);
        }
        if (ok) {
            CUtensorMap* dst = reinterpret_cast<CUtensorMap*>(base + tmap_off);
            cudaMemcpy(dst, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice);
            w.tmaps = dst;
        }
    }
    cudaMemset(w.ctr, 0, (size_t)kCtrCount * 8);
    cudaMemset(w.status, 0, 4);
    dec->status_host = nullptr;
    dec->status_ev = nullptr;
    dec->status_pending = false;
    dec->sync = 0;
    if ((e = cudaHostAlloc(reinterpret_cast<void**>(&dec->status_host), 4, cudaHostAllocDefault)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&dec->status_ev, cudaEventDisableTiming)) != cudaSuccess) {
        const std::string msg = std::string("decoder status mirror: ") + cudaGetErrorString(e);
        if (dec->status_host) cudaFreeHost(dec->status_host);
        cudaFree(dec->block);
        delete dec;
        return fail(ZHA_ERR_CUDA, msg);
    }
    *dec->status_host = 0;
    *out = dec;
    return ZHA_OK;
}

extern "C" zha_status zha_decoder_destroy(zha_decoder* dec) {
    if (!dec) return ZHA_OK;
    cudaDeviceSynchronize();
    cudaFree(dec->block);
    if (dec->status_ev) cudaEventDestroy(dec->status_ev);
    if (dec->status_host) cudaFreeHost(dec->status_host);
    delete dec;
    return ZHA_OK;
}

// Text of the device status bits for an error message.
static std::string status_text(int32_t st) {
    std::string t;
    char buf[32];
    snprintf(buf, sizeof(buf), "device status 0x%x:", (unsigned)st);
    t = buf;
    if (st & kStatusSelectFallbackLimit) t += " top-p select ran out of bisection steps;";
    if (st & kStatusCapacity) t += " a union list reached its capacity;";
    if (st & kStatusTimeout) t += " a tensor-core pipeline wait gave up;";
    if (st & kStatusRange) t += " an input or summary outside the fp16 range reached the tensor-core scorer;";
    if (st & kStatusShardKeys) t += " a sharded cut's boundary bin held more keys than the ranks can exchange;";
    return t;
}

// Start of a routing / attention call: a completed earlier call whose status word was not
// 0 is reported now (once), and nothing of this call is enqueued.
static zha_status check_previous(zha_decoder* dec) {
    if (!dec->status_pending) return ZHA_OK;
    const cudaError_t before = cudaPeekAtLastError();
    const cudaError_t q = cudaEventQuery(dec->status_ev);
    if (q == cudaErrorNotReady) {
        // "not ready" is not a failure: if the query left it as the thread's last error,
        // clear it (and nothing that was there before)
        if (before == cudaSuccess && cudaPeekAtLastError() == cudaErrorNotReady) (void)cudaGetLastError();
        return ZHA_OK;              // still running: a later call (or zha_decoder_stats) reports it
    }
    dec->status_pending = false;
    if (q != cudaSuccess) return fail(ZHA_ERR_CUDA, std::string("cudaEventQuery: ") + cudaGetErrorString(q));
    const int32_t st = *dec->status_host;
    if (st) return fail(ZHA_ERR_DEVICE, "an earlier call on this decoder finished with " + status_text(st));
    return ZHA_OK;
}

// End of a routing / attention call: the status word is copied to the host mirror behind
// the call's kernels.  In synchronous mode the call waits for it and reports it.
static zha_status finish_call(zha_decoder* dec, cudaStream_t st) {
    ZHA_CUDA(cudaMemcpyAsync(dec->status_host, dec->w.status, 4, cudaMemcpyDeviceToHost, st));
    ZHA_CUDA(cudaEventRecord(dec->status_ev, st));
    dec->status_pending = true;
    if (!dec->sync) return ZHA_OK;
    ZHA_CUDA(cudaEventSynchronize(dec->status_ev));
    dec->status_pending = false;
    const int32_t s = *dec->status_host;
    if (s) return fail(ZHA_ERR_DEVICE, status_text(s));
    return ZHA_OK;
}

static zha_status fill_seqs(zha_decoder* dec, const void* const* K, const void* const* V) {
    for (int s = 0; s < dec->n_seq; ++s) {
        const zha_tree* t = dec->trees[s];
        if (!t->built) return fail(ZHA_ERR_STATE, "a tree of the decoder has not been built");
        if (t->n_tokens < 1) return fail(ZHA_ERR_STATE, "a tree of the decoder holds no tokens");
        SeqDev& sd = dec->seq_host[s];
        memset(&sd, 0, sizeof(sd));
        sd.C = t->g.C;
        sd.L = t->g.L;
        sd.R = t->g.R;
        sd.ns = t->ns;
        sd.fmt = t->g.format;
        sd.N = t->n_tokens;
        sd.top = ipow(t->g.C, t->g.L);
        sd.T = sd.N / sd.top;
        sd.ld = t->g.capacity;
        for (int l = 1; l <= t->g.L; ++l) {
            sd.n[l] = sd.N / ipow(t->g.C, l);
            sd.cap[l] = t->cap[l];
            sd.rec[l] = t->rec[l];
        }
        sd.rflag = t->rflag;
        sd.no_sink = (dec->sh_world > 0 && dec->sh_tok0 != 0) ? 1 : 0;
        if (K) sd.K = static_cast<const __nv_bfloat16*>(K[s]);
        if (V) sd.V = static_cast<const __nv_bfloat16*>(V[s]);
    }
    return ZHA_OK;
}

static Batch make_batch(const zha_decoder* dec, const void* Q, int32_t n_q, float p) {
    Batch b;
    b.seqs = dec->seq_dev;
    b.n_seq = dec->n_seq;
    b.n_q = n_q;
    b.Hq = dec->Hq;
    b.Hkv = dec->Hkv;
    b.G = dec->G;
    b.d = dec->d;
    b.n_gl = n_q * dec->G;
    b.n_lanes = dec->n_seq * n_q * dec->Hq;
    b.n_groups = dec->n_seq * dec->Hkv;
    b.Q = static_cast<const __nv_bfloat16*>(Q);
    b.p = p;
    b.score_path = dec->score_path;
    b.attn_path = dec->attn_path;
    b.all_r16 = dec->all_r16;
    b.fmt = dec->trees[0]->g.format;
    b.split_tok = attn_on_tensor_cores(b) ? split_tokens(b.n_gl) : decoder_split_tokens(b.n_gl);
    return b;
}

// Checks of a routing call and the reset of its workspace (kept bitmaps, counters, status,
// frontier maxima and sizes).
static zha_status route_prepare(zha_decoder* dec, const void* Q, int32_t n_q, float p, cudaStream_t st) {
    if (!Q || !aligned16(Q)) return fail(ZHA_ERR_ARG, "Q must be a 16-byte aligned device pointer");
    if (n_q < 1 || n_q > dec->max_q) return fail(ZHA_ERR_CAPACITY, "n_q must be in [1, max_queries]");
    if (!(p > 0.0f) || isnan(p)) return fail(ZHA_ERR_ARG, "p must be > 0");
    zha_status s = fill_seqs(dec, nullptr, nullptr);
    if (s != ZHA_OK) return s;
    ZHA_CUDA(cudaMemcpyAsync(dec->seq_dev, dec->seq_host.data(), sizeof(SeqDev) * dec->n_seq,
                             cudaMemcpyHostToDevice, st));
    const int64_t n_lanes = (int64_t)dec->n_seq * n_q * dec->Hq;
    for (int l = 1; l <= dec->Lmax; ++l)
        ZHA_CUDA(cudaMemsetAsync(dec->w.kept[l], 0, (size_t)n_lanes * dec->w.W[l] * 4, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.ctr, 0, (size_t)kCtrCount * 8, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.status, 0, 4, st));
    // ordered-bits 0 is below every float; counts start at 0
    ZHA_CUDA(cudaMemsetAsync(dec->w.lane_max, 0, (size_t)(kMaxL + 1) * dec->lanes_cap * 4, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.lane_cnt, 0, (size_t)(kMaxL + 1) * dec->lanes_cap * 4, st));
    return ZHA_OK;
}

static zha_status route_impl(zha_decoder* dec, const void* Q, int32_t n_q, float p, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    zha_status s = route_prepare(dec, Q, n_q, p, st);
    if (s != ZHA_OK) return s;
    const Batch b = make_batch(dec, Q, n_q, p);
    const float scale = score_scale(dec->d);
    for (int it = 0; it < dec->Lmax; ++it) {
        if (it > 0) ZHA_CUDA(launch_union(b, dec->w, it, 0, st));
        ZHA_CUDA(launch_score(b, dec->w, it, scale, st));
        // candidates of a lane at level L_s - it: at most that level's complete nodes
        int64_t max_cands = 0;
        for (int sq = 0; sq < dec->n_seq; ++sq) {
            const SeqDev& h = dec->seq_host[sq];
            const int lev = h.L - it;
            if (lev >= 1) max_cands = std::max<int64_t>(max_cands, h.n[lev]);
        }
        ZHA_CUDA(launch_select(b, dec->w, it, max_cands, st));
    }
    dec->routed = true;
    dec->last_n_q = n_q;
    return ZHA_OK;
}

static zha_status refuse_shard(const zha_decoder* dec) {
    if (dec->sh_world > 0) return fail(ZHA_ERR_STATE, "a shard decoder routes through the zha_shard_* calls");
    return ZHA_OK;
}

extern "C" zha_status zha_route(zha_decoder* dec, const void* Q, int32_t n_q, float p, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (refuse_shard(dec) != ZHA_OK) return ZHA_ERR_STATE;
    zha_status s = check_previous(dec);
    if (s != ZHA_OK) return s;
    s = route_impl(dec, Q, n_q, p, stream);
    if (s != ZHA_OK) return s;
    return finish_call(dec, static_cast<cudaStream_t>(stream));
}

static zha_status sparse_attn_impl(zha_decoder* dec, const void* const* K, const void* const* V,
                                   const void* Q, int32_t n_q, float* out, void* stream) {
    if (!dec->routed || n_q != dec->last_n_q) return fail(ZHA_ERR_STATE, "zha_sparse_attn needs a zha_route with the same n_q first");
    if (!K || !V || !Q || !out) return fail(ZHA_ERR_ARG, "K, V, Q and out must be non-NULL");
    if (!aligned16(Q) || !aligned16(out)) return fail(ZHA_ERR_ARG, "Q and out must be 16-byte aligned");
    for (int s = 0; s < dec->n_seq; ++s)
        if (!K[s] || !V[s] || !aligned16(K[s]) || !aligned16(V[s]))
            return fail(ZHA_ERR_ARG, "K[s] and V[s] must be 16-byte aligned device pointers");
    zha_status s = fill_seqs(dec, K, V);
    if (s != ZHA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(cudaMemcpyAsync(dec->seq_dev, dec->seq_host.data(), sizeof(SeqDev) * dec->n_seq,
                             cudaMemcpyHostToDevice, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.ctr + kCtrUnionTokens, 0, 2 * 8, st));
    const Batch b = make_batch(dec, Q, n_q, 1.0f);
    int64_t max_splits = 0;
    for (const SeqDev& sd : dec->seq_host) {
        const int64_t nseg = 1 + sd.n[1] + (std::min<int64_t>(sd.top, sd.N) + sd.C - 1) / sd.C;
        const int64_t segs = batch_segs(b, sd.C);
        max_splits = std::max<int64_t>(max_splits, (nseg + segs - 1) / segs);
    }
    if ((int64_t)b.n_lanes * max_splits > dec->part_slots)
        return fail(ZHA_ERR_CAPACITY, "attention splits exceed workspace");
    Work wc = dec->w;
    wc.s_cap = max_splits;   // partial record of (lane x, split) at x * max_splits + split
    ZHA_CUDA(launch_union(b, wc, 0, 1, st));
    ZHA_CUDA(launch_attn(b, wc, max_splits, score_scale(dec->d), st));
    ZHA_CUDA(launch_combine(b, wc, out, st));
    return ZHA_OK;
}

extern "C" zha_status zha_sparse_attn(zha_decoder* dec, const void* const* K, const void* const* V,
                                      const void* Q, int32_t n_q, float* out, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (refuse_shard(dec) != ZHA_OK) return ZHA_ERR_STATE;
    zha_status s = check_previous(dec);
    if (s != ZHA_OK) return s;
    s = sparse_attn_impl(dec, K, V, Q, n_q, out, stream);
    if (s != ZHA_OK) return s;
    return finish_call(dec, static_cast<cudaStream_t>(stream));
}

extern "C" zha_status zha_dense_attn(zha_decoder* dec, const void* const* K, const void* const* V,
                                     const void* Q, int32_t n_q, float* out, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (refuse_shard(dec) != ZHA_OK) return ZHA_ERR_STATE;
    {
        const zha_status s0 = check_previous(dec);
        if (s0 != ZHA_OK) return s0;
    }
    if (n_q < 1 || n_q > dec->max_q) return fail(ZHA_ERR_CAPACITY, "n_q must be in [1, max_queries]");
    if (!K || !V || !Q || !out) return fail(ZHA_ERR_ARG, "K, V, Q and out must be non-NULL");
    if (!aligned16(Q) || !aligned16(out)) return fail(ZHA_ERR_ARG, "Q and out must be 16-byte aligned");
    for (int s = 0; s < dec->n_seq; ++s)
        if (!K[s] || !V[s] || !aligned16(K[s]) || !aligned16(V[s]))
            return fail(ZHA_ERR_ARG, "K[s] and V[s] must be 16-byte aligned device pointers");
    zha_status s = fill_seqs(dec, K, V);
    if (s != ZHA_OK) return s;
    // No complete top node: no sink, no routed chunks, every token in the tail that every
    // lane attends.  The next zha_route / zha_sparse_attn uploads the trees' own counts again.
    for (SeqDev& sd : dec->seq_host) sd.T = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(cudaMemcpyAsync(dec->seq_dev, dec->seq_host.data(), sizeof(SeqDev) * dec->n_seq,
                             cudaMemcpyHostToDevice, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.ctr + kCtrUnionTokens, 0, 2 * 8, st));
    ZHA_CUDA(cudaMemsetAsync(dec->w.status, 0, 4, st));
    Batch b = make_batch(dec, Q, n_q, 1.0f);
    b.dense = 1;
    int64_t max_splits = 0;
    for (const SeqDev& sd : dec->seq_host) {
        const int64_t nseg = (sd.N + sd.C - 1) / sd.C;
        const int64_t segs = batch_segs(b, sd.C);
        max_splits = std::max<int64_t>(max_splits, (nseg + segs - 1) / segs);
    }
    if ((int64_t)b.n_lanes * max_splits > dec->part_slots)
        return fail(ZHA_ERR_CAPACITY, "attention splits exceed workspace");
    Work wc = dec->w;
    wc.s_cap = max_splits;
    ZHA_CUDA(launch_attn(b, wc, max_splits, score_scale(dec->d), st));
    ZHA_CUDA(launch_combine(b, wc, out, st));
    return finish_call(dec, st);
}

extern "C" zha_status zha_decode(zha_decoder* dec, const void* const* K, const void* const* V,
                                 const void* Q, int32_t n_q, float p, float* out, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (refuse_shard(dec) != ZHA_OK) return ZHA_ERR_STATE;
    zha_status s = check_previous(dec);
    if (s != ZHA_OK) return s;
    s = route_impl(dec, Q, n_q, p, stream);
    if (s != ZHA_OK) return s;
    s = sparse_attn_impl(dec, K, V, Q, n_q, out, stream);
    if (s != ZHA_OK) return s;
    return finish_call(dec, static_cast<cudaStream_t>(stream));
}


// ------------------------------------------------------------------------------ sharded sequence
static_assert(ZHA_SHARD_BINS == kShardBins && ZHA_SHARD_KEYS == kShardKeys, "exchange sizes of zha.h");
static_assert(kStatusShardKeys == 16, "status bit of zha.h");
//
// One sequence split over ranks: each level's cut over the union of the ranks' frontiers,
// taken by k_select in three phases around the caller's collectives (histogram out; cut on
// the summed histogram with the boundary keys out; finish on every rank's keys).

extern "C" zha_status zha_shard_decoder_create(const zha_tree* tree, int32_t max_queries, int32_t rank,
                                               int32_t world, int64_t token_offset, zha_decoder** out) {
    if (!tree) return fail(ZHA_ERR_ARG, "tree is NULL");
    if (!out) return fail(ZHA_ERR_ARG, "out is NULL");
    if (world < 1 || rank < 0 || rank >= world) return fail(ZHA_ERR_ARG, "rank must be in [0, world)");
    const int64_t top = ipow(tree->g.C, tree->g.L);
    if (token_offset < 0 || token_offset % top != 0)
        return fail(ZHA_ERR_ARG, "token_offset must be a non-negative multiple of C^L");
    if ((rank == 0) != (token_offset == 0)) return fail(ZHA_ERR_ARG, "rank 0, and only rank 0, starts at token 0");
    const zha_tree* one[1] = {tree};
    zha_decoder* dec = nullptr;
    const zha_status s = zha_decoder_create(one, 1, max_queries, &dec);
    if (s != ZHA_OK) return s;
    dec->sh_rank = rank;
    dec->sh_world = world;
    dec->sh_tok0 = token_offset;
    dec->sh_step = -1;
    *out = dec;
    return ZHA_OK;
}

// The protocol position a call must find, and the exchange pointers it uses.
static zha_status shard_check(const zha_decoder* dec, int32_t level, int step, const zha_shard_exchange* ex) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (dec->sh_world < 1) return fail(ZHA_ERR_STATE, "not a shard decoder (zha_shard_decoder_create)");
    if (dec->sh_step != step || dec->sh_level != level)
        return fail(ZHA_ERR_STATE, "sharded decode call out of order (see the protocol in zha.h)");
    if (!ex) return fail(ZHA_ERR_ARG, "exchange is NULL");
    auto ok = [](const void* q) { return q && aligned16(q); };
    bool good = true;
    switch (step) {
        case 0: case 1: good = ok(ex->lane_max) && ok(ex->lane_cnt) && (step == 0 || ok(ex->hist)); break;
        case 2: good = ok(ex->hist) && ok(ex->keys) && ok(ex->nkeys); break;
        case 3: good = ok(ex->keys_all) && ok(ex->nkeys_all); break;
        case 4: good = ok(ex->out) && ok(ex->lse); break;
        case 5: good = ok(ex->out_all) && ok(ex->lse_all); break;
        default: break;
    }
    if (!good) return fail(ZHA_ERR_ARG, "an exchange buffer this step uses is NULL or not 16-byte aligned");
    return ZHA_OK;
}

extern "C" zha_status zha_shard_begin(zha_decoder* dec, const void* Q, int32_t n_q, float p, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (dec->sh_world < 1) return fail(ZHA_ERR_STATE, "not a shard decoder (zha_shard_decoder_create)");
    const zha_tree* t = dec->trees[0];
    const int64_t top = ipow(t->g.C, t->g.L);
    if (t->built && dec->sh_rank < dec->sh_world - 1 && t->n_tokens % top != 0)
        return fail(ZHA_ERR_STATE, "every shard but the last must hold a multiple of C^L tokens");
    if (t->built && (dec->sh_tok0 + t->n_tokens) / t->g.C > (int64_t(1) << 24))
        return fail(ZHA_ERR_CAPACITY, "a sharded sequence holds at most 2^24 level-1 nodes");
    zha_status s = check_previous(dec);
    if (s != ZHA_OK) return s;
    s = route_prepare(dec, Q, n_q, p, static_cast<cudaStream_t>(stream));
    if (s != ZHA_OK) return s;
    dec->sh_Q = Q;
    dec->sh_nq = n_q;
    dec->sh_p = p;
    dec->sh_level = t->g.L;
    dec->sh_step = 0;
    dec->routed = false;
    return ZHA_OK;
}

// Work of one select phase of the sharded cut at `level`.
static Work shard_work(const zha_decoder* dec, int phase, int32_t level, const zha_shard_exchange* ex) {
    Work w = dec->w;
    const zha_tree* t = dec->trees[0];
    w.sh_phase = phase;
    w.sh_world = dec->sh_world;
    w.sh_off = dec->sh_tok0 / ipow(t->g.C, level);
    w.sh_hist = reinterpret_cast<unsigned long long*>(ex->hist);
    w.sh_keys = reinterpret_cast<unsigned long long*>(ex->keys);
    w.sh_nkeys = ex->nkeys;
    w.sh_keys_all = reinterpret_cast<const unsigned long long*>(ex->keys_all);
    w.sh_nkeys_all = ex->nkeys_all;
    w.sh_need = dec->sh_need;
    return w;
}

extern "C" zha_status zha_shard_score(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream) {
    zha_status s = shard_check(dec, level, 0, ex);
    if (s != ZHA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Batch b = make_batch(dec, dec->sh_Q, dec->sh_nq, dec->sh_p);
    const int it = dec->trees[0]->g.L - level;
    if (it > 0) ZHA_CUDA(launch_union(b, dec->w, it, 0, st));
    ZHA_CUDA(launch_score(b, dec->w, it, score_scale(dec->d), st));
    ZHA_CUDA(launch_shard_lanes(dec->w.lane_max + (int64_t)level * dec->w.lanes_cap,
                                dec->w.lane_cnt + (int64_t)level * dec->w.lanes_cap, ex->lane_max, ex->lane_cnt,
                                b.n_lanes, true, st));
    dec->sh_step = 1;
    return ZHA_OK;
}

// One select phase (1, 2 or 3) of the sharded cut at `level`.
static zha_status shard_select(zha_decoder* dec, int32_t level, int phase, const zha_shard_exchange* ex,
                               cudaStream_t st) {
    const Batch b = make_batch(dec, dec->sh_Q, dec->sh_nq, dec->sh_p);
    const int it = dec->trees[0]->g.L - level;
    const Work w = shard_work(dec, phase, level, ex);
    ZHA_CUDA(launch_select(b, w, it, dec->seq_host[0].n[level], st));
    return ZHA_OK;
}

extern "C" zha_status zha_shard_hist(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream) {
    zha_status s = shard_check(dec, level, 1, ex);
    if (s != ZHA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the frontier maxima and sizes over all ranks back into the decoder's arrays
    ZHA_CUDA(launch_shard_lanes(dec->w.lane_max + (int64_t)level * dec->w.lanes_cap,
                                dec->w.lane_cnt + (int64_t)level * dec->w.lanes_cap, ex->lane_max, ex->lane_cnt,
                                (int64_t)dec->sh_nq * dec->Hq, false, st));
    s = shard_select(dec, level, 1, ex, st);
    if (s != ZHA_OK) return s;
    dec->sh_step = 2;
    return ZHA_OK;
}

extern "C" zha_status zha_shard_cut(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream) {
    zha_status s = shard_check(dec, level, 2, ex);
    if (s != ZHA_OK) return s;
    s = shard_select(dec, level, 2, ex, static_cast<cudaStream_t>(stream));
    if (s != ZHA_OK) return s;
    dec->sh_step = 3;
    return ZHA_OK;
}

extern "C" zha_status zha_shard_finish(zha_decoder* dec, int32_t level, const zha_shard_exchange* ex, void* stream) {
    zha_status s = shard_check(dec, level, 3, ex);
    if (s != ZHA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = shard_select(dec, level, 3, ex, st);
    if (s != ZHA_OK) return s;
    if (level > 1) {
        dec->sh_level = level - 1;
        dec->sh_step = 0;
        return ZHA_OK;
    }
    dec->sh_level = 0;
    dec->sh_step = 4;
    dec->routed = true;
    dec->last_n_q = dec->sh_nq;
    return finish_call(dec, st);
}

extern "C" zha_status zha_shard_attend(zha_decoder* dec, const void* K, const void* V, const zha_shard_exchange* ex,
                                       void* stream) {
    zha_status s = shard_check(dec, 0, 4, ex);
    if (s != ZHA_OK) return s;
    s = check_previous(dec);
    if (s != ZHA_OK) return s;
    const void* Ks[1] = {K};
    const void* Vs[1] = {V};
    dec->w.lse_out = ex->lse;
    s = sparse_attn_impl(dec, Ks, Vs, dec->sh_Q, dec->sh_nq, ex->out, stream);
    dec->w.lse_out = nullptr;
    if (s != ZHA_OK) return s;
    dec->sh_step = 5;
    return ZHA_OK;
}

extern "C" zha_status zha_shard_combine(zha_decoder* dec, const zha_shard_exchange* ex, float* out, void* stream) {
    zha_status s = shard_check(dec, 0, 5, ex);
    if (s != ZHA_OK) return s;
    if (!out || !aligned16(out)) return fail(ZHA_ERR_ARG, "out must be a 16-byte aligned device pointer");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(launch_shard_combine(ex->out_all, ex->lse_all, (int64_t)dec->sh_nq * dec->Hq, dec->sh_world, dec->d,
                                  out, st));
    dec->sh_step = -1;
    return finish_call(dec, st);
}

extern "C" zha_status zha_decoder_set_sync(zha_decoder* dec, int32_t on) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    dec->sync = on ? 1 : 0;
    return ZHA_OK;
}

extern "C" zha_status zha_decoder_set_kernels(zha_decoder* dec, int32_t score, int32_t attn) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    auto ok = [](int32_t v) { return v == ZHA_KERNELS_AUTO || v == ZHA_KERNELS_SIMT || v == ZHA_KERNELS_TENSOR; };
    if (!ok(score) || !ok(attn)) return fail(ZHA_ERR_ARG, "unknown kernel choice");
    if (score == ZHA_KERNELS_TENSOR && !dec->all_r16)
        return fail(ZHA_ERR_ARG, "the tensor-core scorer needs R = 16 in every tree");
    if (score == ZHA_KERNELS_TENSOR && dec->trees[0]->g.format == ZHA_SUMMARY_FP4)
        return fail(ZHA_ERR_ARG, "MXFP4 records are scored on the CUDA cores only");
    if (score == ZHA_KERNELS_TENSOR && !dec->w.tmaps)
        return fail(ZHA_ERR_CUDA, "the tensor-core scorer's TMA maps could not be encoded");
    dec->score_path = score;
    dec->attn_path = attn;
    return ZHA_OK;
}

extern "C" int64_t zha_decoder_words(const zha_decoder* dec, int32_t level) {
    if (!dec || level < 1 || level > dec->Lmax) return 0;
    return dec->w.W[level];
}

extern "C" zha_status zha_decoder_export_kept(const zha_decoder* dec, int32_t level, uint32_t* bits,
                                              int32_t* counts, void* stream) {
    if (!dec) return fail(ZHA_ERR_ARG, "decoder is NULL");
    if (!dec->routed) return fail(ZHA_ERR_STATE, "no zha_route yet");
    if (level < 1 || level > dec->Lmax) return fail(ZHA_ERR_ARG, "level out of range");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n_lanes = (int64_t)dec->n_seq * dec->last_n_q * dec->Hq;
    if (bits)
        ZHA_CUDA(cudaMemcpyAsync(bits, dec->w.kept[level], (size_t)n_lanes * dec->w.W[level] * 4,
                                 cudaMemcpyDeviceToDevice, st));
    if (counts) {
        // Lanes of trees with fewer levels never write their count at this level.
        for (int s = 0; s < dec->n_seq; ++s) {
            const int64_t l0 = (int64_t)s * dec->last_n_q * dec->Hq, nl = (int64_t)dec->last_n_q * dec->Hq;
            if (level <= dec->trees[s]->g.L)
                ZHA_CUDA(cudaMemcpyAsync(counts + l0, dec->w.kcount + (int64_t)level * dec->lanes_cap + l0,
                                         (size_t)nl * 4, cudaMemcpyDeviceToDevice, st));
            else
                ZHA_CUDA(cudaMemsetAsync(counts + l0, 0, (size_t)nl * 4, st));
        }
    }
    return ZHA_OK;
}

extern "C" zha_status zha_decoder_stats(const zha_decoder* dec, zha_decode_stats* out, void* stream) {
    if (!dec || !out) return fail(ZHA_ERR_ARG, "decoder or out is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned long long ctr[kCtrCount];
    int32_t status = 0;
    ZHA_CUDA(cudaMemcpyAsync(ctr, dec->w.ctr, sizeof(ctr), cudaMemcpyDeviceToHost, st));
    ZHA_CUDA(cudaMemcpyAsync(&status, dec->w.status, 4, cudaMemcpyDeviceToHost, st));
    ZHA_CUDA(cudaStreamSynchronize(st));
    if (dec->status_pending && cudaEventQuery(dec->status_ev) == cudaSuccess)
        const_cast<zha_decoder*>(dec)->status_pending = false;   // reported here instead
    memset(out, 0, sizeof(*out));
    for (int l = 1; l <= kMaxL; ++l) {
        out->union_nodes[l - 1] = (int64_t)ctr[kCtrUnionNodes + l];
        out->lane_nodes[l - 1] = (int64_t)ctr[kCtrLaneNodes + l];
    }
    out->union_tokens = (int64_t)ctr[kCtrUnionTokens];
    out->lane_tokens = (int64_t)ctr[kCtrLaneTokens];
    const zha_geometry& g = dec->trees[0]->g;
    out->node_bytes = scored_node_bytes(g.R, g.d, g.format);
    out->status = status;
    return status ? fail(ZHA_ERR_DEVICE, "device status word is set") : ZHA_OK;
}
