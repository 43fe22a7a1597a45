// zha_route.cu - top-down top-p routing kernels.
//
// What is computed (pages: fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的 —
// score the top level, keep the fewest nodes whose estimated mass reaches the fraction p, then
// descend one level at a time; wqu.guru, section "How does top-p routing pick tokens?"): for every lane (query token, query head h, KV head
// g = h*Hkv/Hq) and level l from L down to 1, each frontier node j gets the plane estimate
//     e_j = max_r ( s q.m_r(j) + b_r(j) ),
// the frontier's softmax masses P_j = exp(e_j - max e) / sum exp(e - max e) are ordered by
// (e desc, j asc), and the shortest prefix with cumulative mass >= p is kept (p >= 1 keeps
// all).  The next frontier is the C children of each kept node.
//
// One level of one launch covers every lane of the batch:
//   k_union  - per (sequence, KV head) group: sorted union of the lanes' kept nodes of the
//              previous level (their children are the group's candidates);
//   k_score  - each candidate node record (m, b) is read once per group and scored against
//              all of the group's lanes (GQA heads and query tokens share the read);
//   k_select - per lane: deterministic top-p cut (fixed-point masses, radix-style bins on
//              max e - e, exact (e, j) ordering inside the boundary bin), kept bitmap out.
#include <math.h>

#include <type_traits>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr unsigned kFull = 0xffffffffu;

// ----------------------------------------------------------------------------- block helpers

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Block-wide reductions; `red` holds >= 32 elements; all threads get the result.
template <typename T>
__device__ T block_sum(T v, T* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    T t = (lane < nw) ? red[lane] : T(0);
    t = warp_sum(t);
    return t;
}

template <typename T>
__device__ __forceinline__ T block_min_t(T v, T* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const T u = __shfl_xor_sync(kFull, v, o);
        v = u < v ? u : v;
    }
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    T t = (lane < nw) ? red[lane] : red[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const T u = __shfl_xor_sync(kFull, t, o);
        t = u < t ? u : t;
    }
    return t;
}

template <typename T>
__device__ __forceinline__ T block_max_t(T v, T* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const T u = __shfl_xor_sync(kFull, v, o);
        v = u > v ? u : v;
    }
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    T t = (lane < nw) ? red[lane] : red[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const T u = __shfl_xor_sync(kFull, t, o);
        t = u > t ? u : t;
    }
    return t;
}

// Block-wide exclusive scan; red holds >= 33 elements; total returned through `total`.
template <typename T>
__device__ T block_excl_scan(T v, T* red, T& total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    T incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) red[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const T ws = lane < nw ? red[lane] : T(0);
        T wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const T t = __shfl_up_sync(kFull, wi, o);
            if (lane >= o) wi += t;
        }
        red[lane] = wi - ws;
        if (lane == 31) red[32] = wi;
    }
    __syncthreads();
    total = red[32];
    return red[wid] + incl - v;
}

// ----------------------------------------------------------------------------- union

// Level whose kept sets a union call gathers for sequence sq, 0 if none.  Mode 0: routing
// iteration it >= 1 needs the kept nodes of level L_s - it + 1 (their children are the
// candidates); mode 1: attention needs the kept level-1 chunks.
__device__ __forceinline__ int union_level(const SeqDev& sq, int it, int mode) {
    if (mode == 0) {
        const int lev = sq.L - it;
        return (it == 0 || lev < 1) ? 0 : lev + 1;
    }
    return sq.T == 0 ? 0 : 1;
}

// Nodes of level ulev that may enter a union: every complete node when routing; for
// attention only the level-1 chunks under complete top nodes (T C^L / C of them).  Chunks
// at or after the first tail token are attended as tail anyway, and bits past the complete
// chunks name no rows: bits set there in a caller's bitmap are ignored.
__device__ __forceinline__ int64_t union_limit(const SeqDev& sq, int ulev, int mode) {
    return mode == 1 ? sq.T * (sq.top / sq.C) : sq.n[ulev];
}

// OR of the kept bitmaps of a chunk of a group's lanes into the group's union bitmap.
// Grid: (word blocks, lane chunks of `lanes_per_block`, groups).
__global__ void __launch_bounds__(256) k_union_or(Batch b, Work w, int it, int mode, int lanes_per_block) {
    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int ulev = union_level(sq, it, mode);
    if (ulev == 0) return;
    const int64_t lim = union_limit(sq, ulev, mode);
    const int64_t nwords = (lim + 31) / 32;
    const int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (wi >= nwords) return;
    const int y0 = blockIdx.y * lanes_per_block;
    const int y1 = min(b.n_gl, y0 + lanes_per_block);
    const uint32_t* kb = w.kept[ulev];
    const int64_t W = w.W[ulev];
    uint32_t word = 0;
#pragma unroll 8
    for (int y = y0; y < y1; ++y) word |= __ldg(kb + lane_of(b, s, g, y) * W + wi);
    const int64_t rest = lim - wi * 32;          // valid bits of this word (>= 1)
    if (rest < 32) word &= (1u << rest) - 1u;
    if (word) atomicOr(w.uword + (int64_t)grp * w.uw + wi, word);
}

// Compacts a group's union bitmap into the sorted list of set bits.  Grid (chunks, groups):
// block c writes the entries of words [c kCompactWords, (c + 1) kCompactWords); its offset in
// the list is the number of set bits in the words before its chunk, which the block counts
// itself (at most a few tens of KB from L2), so one launch suffices and every chunk is written
// in parallel (each thread one word: at most 32 entries).  The block holding the group's last
// word writes the count.
constexpr int kCompactThreads = 256;
constexpr int kCompactWords = 256;

__global__ void __launch_bounds__(kCompactThreads) k_union_compact(Batch b, Work w, int it, int mode) {
    __shared__ int red[33];
    const int grp = blockIdx.y;
    const int s = grp / b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int ulev = union_level(sq, it, mode);
    if (ulev == 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            w.ucount[grp] = 0;
            if (mode == 1) atomicAdd(&w.ctr[kCtrUnionTokens], (unsigned long long)sq.N);   // dense: A = [0, N)
        }
        return;
    }
    const int64_t nwords = (union_limit(sq, ulev, mode) + 31) / 32;
    const int64_t c0 = (int64_t)blockIdx.x * kCompactWords;
    if (c0 >= nwords && !(nwords == 0 && blockIdx.x == 0)) return;   // whole block, before any barrier
    const uint32_t* uwp = w.uword + (int64_t)grp * w.uw;
    int32_t* out = w.ulist + (int64_t)grp * w.us;
    // set bits before this chunk
    int pre = 0;
    for (int64_t wi = threadIdx.x; wi < c0; wi += kCompactThreads) pre += __popc(uwp[wi]);
    int base = block_sum<int>(pre, red);
    const int64_t c1 = c0 + kCompactWords < nwords ? c0 + kCompactWords : nwords;
    for (int64_t w0 = c0; w0 < c1; w0 += kCompactThreads) {
        const int64_t wi = w0 + threadIdx.x;
        uint32_t word = wi < c1 ? uwp[wi] : 0u;
        int total;
        const int excl = block_excl_scan<int>(__popc(word), red, total);
        int k = base + excl;
        while (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            if (k < w.us) out[k] = (int32_t)(wi * 32 + bit);   // the list never outgrows its row
            ++k;
        }
        base += total;
    }
    if (c1 < nwords) return;                                   // not the group's last chunk
    if (base > w.us) {                                         // cannot happen with the limit above
        if (threadIdx.x == 0) atomicOr(w.status, kStatusCapacity);
        base = (int)w.us;
    }
    if (threadIdx.x == 0) {
        w.ucount[grp] = base;
        if (mode == 1) {
            // attended tokens of the group: sink + kept chunks (token 0 once) + tail; a later
            // shard of a sharded sequence has no sink and attends its token 0 with chunk 0
            const int64_t tail = sq.N - sq.T * sq.top;
            const int has0 = nwords > 0 ? (int)(uwp[0] & 1u) : 0;
            const int64_t s0 = sq.no_sink ? 0 : 1;
            atomicAdd(&w.ctr[kCtrUnionTokens], (unsigned long long)(tail + s0 + (int64_t)base * sq.C - s0 * has0));
        }
    }
}

// ----------------------------------------------------------------------------- score

// Warp = 8 lanes x 4 quarter-threads; thread (lane, quarter) keeps its lane's query
// dimensions {16 i + 4 quarter + c} in registers.  WB warps split a block of 8*WB lanes,
// 8/WB node slots run concurrently.  Each node record is read with 16-byte loads.
template <int D, int FMT>
__global__ void __launch_bounds__(256) k_score(Batch b, Work w, int it, float scale) {
    constexpr bool BF = FMT == kFmtBf16;
    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int lev = sq.L - it;
    if (lev < 1) return;
    const bool top = (lev == sq.L);
    const int C = sq.C;
    const int64_t nc = top ? sq.T : (int64_t)w.ucount[grp] * C;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        atomicAdd(&w.ctr[kCtrUnionNodes + lev], (unsigned long long)nc);
        tree_flag_status(*sq.rflag, w.status);
    }
    if (nc == 0) return;
    const int WB = min(8, (b.n_gl + 7) / 8);
    const int NPC = 8 / WB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= WB * NPC) return;
    const int lb = warp % WB, slot = warp / WB;
    const int y = (blockIdx.y * WB + lb) * 8 + (lane >> 2);
    const int q = lane & 3;
    const bool lane_ok = y < b.n_gl;
    const int64_t x = lane_of(b, s, g, lane_ok ? y : 0);

    float qv[D / 4];
    {
        const uint2* p = reinterpret_cast<const uint2*>(b.Q + x * D);
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const uint2 u = __ldg(p + 4 * i + q);
            const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
            const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
            qv[4 * i] = a0.x; qv[4 * i + 1] = a0.y; qv[4 * i + 2] = a1.x; qv[4 * i + 3] = a1.y;
        }
    }
    const int R = sq.R;
    const int64_t ns = sq.ns;
    const float* base = sq.rec[lev] + (int64_t)g * sq.cap[lev] * ns;
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    float* ex = w.e + x * w.es;
    // the lane's kept set one level up decides which candidates are on its frontier
    const uint32_t* Pb = top ? nullptr : w.kept[lev + 1] + x * w.W[lev + 1];
    float fmax = -INFINITY;
    int fcnt = 0;
    for (int64_t k = (int64_t)blockIdx.x * NPC + slot; k < nc; k += (int64_t)gridDim.x * NPC) {
        const int64_t j = top ? k : (int64_t)__ldg(ul + k / C) * C + k % C;
        const float* rec = base + j * ns;
        const __half* rh = reinterpret_cast<const __half*>(rec);
        float best = -INFINITY;
        const float* brow = rec + b_offset(R, D, FMT);
        for (int r = 0; r < R; ++r) {
            const uint2* hrow = reinterpret_cast<const uint2*>(rh + (int64_t)r * D);   // also the bf16 plane
            const uint2* lrow = reinterpret_cast<const uint2*>(rh + (int64_t)R * D + (int64_t)r * D);
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                float4 m;
                if constexpr (FMT == kFmtFp4) {
                    m = fp4_load4(rec, R, D, r, 16 * i + 4 * q);
                } else if constexpr (BF) {
                    const uint2 hv = __ldg(hrow + 4 * i + q);
                    const float2 m01 = m_decode_bf16(hv.x), m23 = m_decode_bf16(hv.y);
                    m = make_float4(m01.x, m01.y, m23.x, m23.y);
                } else {
                    const uint2 hv = __ldg(hrow + 4 * i + q), lv = __ldg(lrow + 4 * i + q);
                    const float2 m01 = m_decode2(hv.x, lv.x), m23 = m_decode2(hv.y, lv.y);
                    m = make_float4(m01.x, m01.y, m23.x, m23.y);
                }
                dot = fmaf(qv[4 * i], m.x, dot);
                dot = fmaf(qv[4 * i + 1], m.y, dot);
                dot = fmaf(qv[4 * i + 2], m.z, dot);
                dot = fmaf(qv[4 * i + 3], m.w, dot);
            }
            dot += __shfl_xor_sync(kFull, dot, 1);
            dot += __shfl_xor_sync(kFull, dot, 2);
            best = fmaxf(best, fmaf(scale, dot, __ldg(brow + r)));
        }
        if (lane_ok && q == 0) {
            bool mb = true;
            if (!top) {
                const int64_t pj = j / C;
                mb = (__ldg(Pb + (pj >> 5)) >> (pj & 31)) & 1u;
            }
            ex[k] = mb ? best : -INFINITY;   // candidate order
            if (mb) {
                fmax = fmaxf(fmax, best);
                ++fcnt;
            }
        }
    }
    if (lane_ok && q == 0 && fcnt > 0) {
        atomicMax(w.lane_max + (int64_t)lev * w.lanes_cap + x, ord_bits(fmax));
        atomicAdd(w.lane_cnt + (int64_t)lev * w.lanes_cap + x, fcnt);
    }
}

// Scorer for groups of at most kFewLanes lanes with R = 16 (one or two query tokens): one
// warp per candidate node reads the node's whole record at once - thread t holds half of
// plane row r = t / 2 (dims (t % 2) D/2 ..), D/16 16-byte loads per fp16 plane, all issued
// together, so a node costs one DRAM round trip - decodes m = hi + lo once and scores every
// lane of the group from it (the lanes' query rows in shared memory).  The same estimate as
// k_score: e = max_r (s q.m_r + b_r), -inf off the lane's frontier, in candidate order.
constexpr int kFewLanes = 16;

template <int D, int FMT>
__global__ void __launch_bounds__(256, 2) k_score_few(Batch b, Work w, int it, float scale) {
    constexpr bool BF = FMT == kFmtBf16;
    constexpr int kHalf = D / 2;      // dims per thread
    constexpr int kV = kHalf / 8;     // 16-byte pieces per plane per thread
    constexpr int kRow = kHalf + 4;   // shared row stride of a query half (the two halves of a
                                      // row fall in different banks)
    __shared__ __align__(16) float sqy[kFewLanes][2][kRow];
    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int lev = sq.L - it;
    if (lev < 1) return;
    const bool top = (lev == sq.L);
    const int C = sq.C;
    const int64_t nc = top ? sq.T : (int64_t)w.ucount[grp] * C;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        atomicAdd(&w.ctr[kCtrUnionNodes + lev], (unsigned long long)nc);
        tree_flag_status(*sq.rflag, w.status);
    }
    if (nc == 0) return;
    const int nl = b.n_gl;            // <= kFewLanes (checked by the launcher)
    for (int i = threadIdx.x; i < nl * D; i += blockDim.x) {
        const int y = i / D, k = i - y * D;
        sqy[y][k / kHalf][k % kHalf] = __bfloat162float(b.Q[lane_of(b, s, g, y) * D + k]);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 1, hf = lane & 1;
    const int R = sq.R;               // 16
    const int64_t ns = sq.ns;
    const float* base = sq.rec[lev] + (int64_t)g * sq.cap[lev] * ns;
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    // lane y = this thread's lane (threads 0 .. nl-1): its frontier test and statistics
    const int64_t xm = lane_of(b, s, g, lane < nl ? lane : 0);
    const uint32_t* Pb = top ? nullptr : w.kept[lev + 1] + xm * w.W[lev + 1];
    float* ex = w.e + xm * w.es;
    float fmax = -INFINITY;
    int fcnt = 0;
    const int64_t wstep = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t k = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; k < nc; k += wstep) {
        const int64_t j = top ? k : (int64_t)__ldg(ul + k / C) * C + k % C;
        const float* rec = base + j * ns;
        const __half* rh = reinterpret_cast<const __half*>(rec);
        const uint4* hp = reinterpret_cast<const uint4*>(rh + (int64_t)r * D + hf * kHalf);   // also the bf16 plane
        const uint4* lp = reinterpret_cast<const uint4*>(rh + (int64_t)R * D + (int64_t)r * D + hf * kHalf);
        uint4 hv[kV], lv[kV];
        float m[kHalf];
        const float br = __ldg(rec + b_offset(R, D, FMT) + r);
        if constexpr (FMT == kFmtFp4) {
            // this thread's D/2 codes (D/4 bytes) and the scales of their D/64 blocks
            constexpr int kC4 = kHalf / 32;             // 16-byte pieces of codes
            const uint4* cq = reinterpret_cast<const uint4*>(fp4_codes(rec) + ((int64_t)r * D + hf * kHalf) / 2);
            uint4 cv[kC4];
#pragma unroll
            for (int v = 0; v < kC4; ++v) cv[v] = __ldg(cq + v);
            const uint8_t* sc = fp4_scales(rec, R, D) + (int64_t)r * (D / kFp4Block) + hf * (kHalf / kFp4Block);
#pragma unroll
            for (int v = 0; v < kC4; ++v) {
                const float X = fp4_scale(__ldg(sc + v));
                const uint32_t cw[4] = {cv[v].x, cv[v].y, cv[v].z, cv[v].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int t = 0; t < 8; ++t) m[32 * v + 8 * c + t] = fp4_value((cw[c] >> (4 * t)) & 15u, X);
            }
        } else {
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            hv[v] = __ldg(hp + v);
            if constexpr (!BF) lv[v] = __ldg(lp + v);
        }
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const uint32_t hw[4] = {hv[v].x, hv[v].y, hv[v].z, hv[v].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float2 f;
                if constexpr (BF) {
                    f = m_decode_bf16(hw[c]);
                } else {
                    const uint32_t lw[4] = {lv[v].x, lv[v].y, lv[v].z, lv[v].w};
                    f = m_decode2(hw[c], lw[c]);
                }
                m[8 * v + 2 * c] = f.x;
                m[8 * v + 2 * c + 1] = f.y;
            }
        }
        }
        float mine = -INFINITY;
#pragma unroll 1
        for (int y = 0; y < nl; ++y) {
            const float4* q4 = reinterpret_cast<const float4*>(sqy[y][hf]);
            float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
            for (int i = 0; i < kHalf / 4; ++i) {
                const float4 qv = q4[i];
                d0 = fmaf(qv.x, m[4 * i], d0);
                d1 = fmaf(qv.y, m[4 * i + 1], d1);
                d0 = fmaf(qv.z, m[4 * i + 2], d0);
                d1 = fmaf(qv.w, m[4 * i + 3], d1);
            }
            float dot = d0 + d1;
            dot += __shfl_xor_sync(kFull, dot, 1);            // the row's two halves
            float e = fmaf(scale, dot, br);
#pragma unroll
            for (int o = 2; o < 32; o <<= 1) e = fmaxf(e, __shfl_xor_sync(kFull, e, o));   // max over r
            if (lane == y) mine = e;
        }
        if (lane < nl) {
            bool mb = true;
            if (!top) {
                const int64_t pj = j / C;
                mb = (__ldg(Pb + (pj >> 5)) >> (pj & 31)) & 1u;
            }
            ex[k] = mb ? mine : -INFINITY;   // candidate order
            if (mb) {
                fmax = fmaxf(fmax, mine);
                ++fcnt;
            }
        }
    }
    if (lane < nl && fcnt > 0) {
        atomicMax(w.lane_max + (int64_t)lev * w.lanes_cap + xm, ord_bits(fmax));
        atomicAdd(w.lane_cnt + (int64_t)lev * w.lanes_cap + xm, fcnt);
    }
}

// ----------------------------------------------------------------------------- select

constexpr int kSelThreads = 512;
constexpr int kSelThreadsSmall = 128;  // block size when every lane has <= kSelSmallCands candidates
constexpr int64_t kSelSmallCands = 16384;
constexpr int kNB = 2048;            // bins over (max e - e) * kBinScale
constexpr float kBinScale = 64.0f;
constexpr int kCap = 2048;           // boundary-bin candidates sorted in shared memory
static_assert(kShardBins == kNB && kShardKeys == kCap, "the sharded cut exchanges k_select's own bins and keys");
static_assert(kShardMergeKeys * 8 <= kNB * 8 + kCap * 8, "the sharded finish sorts in the histogram and key areas");
constexpr int kUn = 2;               // 128-candidate blocks per warp in flight (gather path)
constexpr int kPD = 4;               // per-thread prefetch ring depth (cp.async), a power of two

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// masses are fixed point with 2^39 for exp(0); sums of <= 2^24 candidates stay below 2^63

// Ascending key order == (e descending, node index ascending).
__device__ __forceinline__ unsigned long long sel_key(float e, int j) {
    return ((unsigned long long)(~ord_bits(e)) << 32) | (unsigned long long)(uint32_t)j;
}
__device__ __forceinline__ float key_score(unsigned long long k) {
    return unord_bits(~(uint32_t)(k >> 32));
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// The cut's arithmetic is shared by every pass and kept off the quarter-rate conversion
// unit: one ex2 per candidate, the rest on the FMA and integer pipes.
// Adds the 64-bit mass (hi, lo) to a bin kept as two 32-bit words: lo into the low word
// (with return, to see its wrap), hi plus the wrap into the high word.  Both atomics are
// predicated (nothing for a zero mass; the second only when it adds something), so the
// update has no branches.
__device__ __forceinline__ void hist_add(uint32_t alo, uint32_t ahi, uint32_t lo, uint32_t hi) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .u32 old, sum, c;\n\t"
        "setp.ne.u32 p, %2, 0;\n\t"
        "mov.u32 old, 0;\n\t"
        "@p atom.shared.add.u32 old, [%0], %3;\n\t"
        "add.u32 sum, old, %3;\n\t"
        "setp.lt.u32 q, sum, old;\n\t"
        "selp.u32 c, 1, 0, q;\n\t"
        "add.u32 c, c, %4;\n\t"
        "setp.ne.and.u32 q, c, 0, p;\n\t"
        "@q red.shared.add.u32 [%1], c;\n\t}\n"
        ::"r"(alo), "r"(ahi), "r"(lo | hi), "r"(lo), "r"(hi)
        : "memory");
}

struct SelMath {
    float nl2M;     // -M log2(e)
    float m64;      // M kBinScale
    // fixed-point mass floor(exp(e - M) 2^39) as 32-bit words (lo, hi): f = exp(e - M) in
    // [0, 1] (flushed to 0 below the normal range) times 2^39 is exact in float32, and its
    // truncation to a 64-bit integer is the floor; one conversion on the otherwise lightly
    // used conversion pipe instead of shifts and selects on the integer pipe
    __device__ __forceinline__ void mass2(float e, uint32_t& lo, uint32_t& hi) const {
        const float f = ex2_approx(fmaf(e, 1.4426950408889634f, nl2M));
        unsigned long long m;
        asm("cvt.rzi.u64.f32 %0, %1;" : "=l"(m) : "f"(f * 549755813888.0f));   // 2^39
        lo = (uint32_t)m;
        hi = (uint32_t)(m >> 32);
    }
    __device__ __forceinline__ unsigned long long mass(float e) const {
        uint32_t lo, hi;
        mass2(e, lo, hi);
        return ((unsigned long long)hi << 32) | lo;
    }
    // bin = round((M - e) kBinScale), clamped to kNB - 1 (magic-number rounding, no conversion)
    __device__ __forceinline__ int bin(float e) const {
        const float t = fminf(fmaf(e, -kBinScale, m64), (float)(kNB - 1));
        return __float_as_int(t + 8388608.0f) - 0x4B000000;
    }
};

// One block per lane.  The scorer left, for every candidate of the lane's group (the
// children of the group's union of kept nodes, or all top nodes) in candidate order, the
// plane estimate if the candidate is on this lane's frontier and -inf otherwise, plus the
// lane's frontier maximum M and size F.  Two passes over the candidates: a histogram of fixed-point masses
// over bins of M - e, then the kept bits of the bins above the boundary bin and the
// boundary bin's candidates, which are sorted by (e desc, j asc) to finish the prefix.
template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) k_select(Batch b, Work w, int it) {
    extern __shared__ unsigned long long sel_smem[];
    // bin masses as two 32-bit words (shared-memory 64-bit atomics are several times slower):
    // hlo accumulates the low words, hhi the high words and every wrap of hlo, so a bin's
    // exact 64-bit mass is hhi 2^32 + hlo
    uint32_t* hlo = reinterpret_cast<uint32_t*>(sel_smem);   // [kNB]
    uint32_t* hhi = hlo + kNB;                                // [kNB]
    unsigned long long* keys = sel_smem + kNB;                // [kCap]
    float4* pref = reinterpret_cast<float4*>(keys + kCap);   // [kPD][threads] prefetched scores
    int32_t* prefj = reinterpret_cast<int32_t*>(pref + (size_t)NT * kPD);   // [kPD][threads] union entries
    auto hist = [&](int i) -> unsigned long long { return ((unsigned long long)hhi[i] << 32) | hlo[i]; };
    __shared__ unsigned long long red_u[33];
    __shared__ int red_i[33];
    __shared__ int s_bstar;
    __shared__ unsigned long long s_cumb;
    __shared__ unsigned int s_nkeys;
    __shared__ int s_found;

    const int64_t x = blockIdx.x;
    const int s = (int)(x / ((int64_t)b.n_q * b.Hq));
    const int g = (int)(x % b.Hq) / b.G;
    const int grp = s * b.Hkv + g;
    const SeqDev& sq = b.seqs[s];
    const int lev = sq.L - it;
    if (lev < 1) return;
    int32_t* kcount = w.kcount + (int64_t)lev * w.lanes_cap + x;
    const int64_t F = w.lane_cnt[(int64_t)lev * w.lanes_cap + x];
    const int phase = w.sh_phase;
    if (threadIdx.x == 0 && phase <= 1) atomicAdd(&w.ctr[kCtrLaneNodes + lev], (unsigned long long)F);
    if (F == 0) {
        if (threadIdx.x == 0 && phase != 3) {
            *kcount = 0;
            if (phase == 2) {
                w.sh_nkeys[x] = 0;
                w.sh_need[x] = 0;
            }
        }
        return;
    }
    if (phase == 1 && !(b.p < 1.0f)) return;      // p >= 1 keeps the whole frontier: no histogram
    const float M = unord_bits(w.lane_max[(int64_t)lev * w.lanes_cap + x]);
    SelMath sm;
    sm.nl2M = -M * 1.4426950408889634f;
    sm.m64 = M * kBinScale;
    const bool top = (lev == sq.L);
    const int C = sq.C;
    // candidate and node indices are < 2^24 (level-1 nodes are capped there): 32-bit math
    const int nu = top ? 0 : w.ucount[grp];
    const int nc = top ? (int)sq.T : nu * C;
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    // candidates 4k..4k+3 are 4 consecutive, 4-aligned nodes
    const bool contig = top || (C % 4 == 0);
    const float* e = w.e + x * w.es;
    uint32_t* outw = w.kept[lev] + x * w.W[lev];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int nblk = (nc + 127) / 128;

    // Sorts kk[0 .. n) by (e desc, j asc) and returns the index of the last key of the
    // shortest prefix whose mass reaches `need` (n - 1 if none does).  Block-uniform.
    auto sort_prefix = [&](unsigned long long* kk, int n, unsigned long long need_) -> int {
        int npow = 1;
        while (npow < n) npow <<= 1;
        for (int i = threadIdx.x; i < npow; i += blockDim.x)
            if (i >= n) kk[i] = ~0ull;
        __syncthreads();
        for (int k = 2; k <= npow; k <<= 1) {
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                for (int i = threadIdx.x; i < npow; i += blockDim.x) {
                    const int ixj = i ^ jj;
                    if (ixj > i) {
                        const unsigned long long a0 = kk[i], a1 = kk[ixj];
                        const bool asc = (i & k) == 0;
                        if ((a0 > a1) == asc) {
                            kk[i] = a1;
                            kk[ixj] = a0;
                        }
                    }
                }
                __syncthreads();
            }
        }
        const int per = (n + blockDim.x - 1) / blockDim.x;
        const int i0 = threadIdx.x * per;
        unsigned long long run = 0;
        for (int i = i0; i < min(n, i0 + per); ++i) run += sm.mass(key_score(kk[i]));
        unsigned long long tot;
        unsigned long long cum = block_excl_scan<unsigned long long>(run, red_u, tot);
        int found = n;
        for (int i = i0; i < min(n, i0 + per); ++i) {
            cum += sm.mass(key_score(kk[i]));
            if (cum >= need_) {
                found = i;
                break;
            }
        }
        found = block_min_t<int>(found, red_i);
        return found >= n ? n - 1 : found;
    };

    if (phase == 3) {
        // sharded cut, last step: every rank's boundary-bin keys (global node ids) for this
        // lane, sorted together; the prefix reaching the needed mass is the same on every
        // rank, and each rank sets the bits of its own nodes
        const unsigned long long need3 = w.sh_need[x];
        if (need3 == 0) return;
        int tot = 0;
        bool over = false;
        for (int r = 0; r < w.sh_world; ++r) {
            const int nr = w.sh_nkeys_all[(int64_t)r * b.n_lanes + x];
            over |= nr > kShardKeys;
            tot += nr;
        }
        if (over || tot > kShardMergeKeys || tot == 0) {
            if (threadIdx.x == 0) atomicOr(w.status, kStatusShardKeys);
            return;
        }
        unsigned long long* kk = sel_smem;                  // the histogram and key areas: 4,096 keys
        int o = 0;
        for (int r = 0; r < w.sh_world; ++r) {
            const int nr = w.sh_nkeys_all[(int64_t)r * b.n_lanes + x];
            const unsigned long long* src = w.sh_keys_all + ((int64_t)r * b.n_lanes + x) * kShardKeys;
            for (int i = threadIdx.x; i < nr; i += blockDim.x) kk[o + i] = src[i];
            o += nr;
        }
        __syncthreads();
        const int found = sort_prefix(kk, tot, need3);
        const int64_t own = sq.n[lev];
        int mine = 0;
        for (int i = threadIdx.x; i <= found; i += blockDim.x) {
            const int64_t jl = (int64_t)(uint32_t)kk[i] - w.sh_off;
            if (jl >= 0 && jl < own) {
                atomicOr(outw + (jl >> 5), 1u << (jl & 31));
                ++mine;
            }
        }
        mine = (int)block_sum<unsigned long long>((unsigned long long)mine, red_u);
        if (threadIdx.x == 0) *kcount += mine;
        return;
    }

    // candidate k -> node index (shifts when C is a power of two)
    const int cs = (C & (C - 1)) == 0 ? __ffs(C) - 1 : -1;
    auto cand_j = [&](int k) -> int {
        if (top) return k;
        if (cs >= 0) return (__ldg(ul + (k >> cs)) << cs) + (k & (C - 1));
        const uint32_t pk = (uint32_t)k / (uint32_t)C;
        return __ldg(ul + pk) * C + (k - (int)pk * C);
    };
    // scores of candidates k0..k0+3 (k0 = 128 bk + 4 lane), stored in candidate order by the
    // scorer; -inf past the end.  With need_j, also the node index of candidate k0 (of the
    // 4 consecutive nodes when contig), loaded independently of the scores.
    auto load = [&](int bk, float4& ev, int& j0, bool need_j) {
        const int k0 = bk * 128 + 4 * lane;
        const bool in = k0 < nc;
        const float4 xv = *reinterpret_cast<const float4*>(e + (in ? k0 : 0));   // rows padded to 128
        j0 = (need_j && in) ? cand_j(k0) : -1;
        ev.x = in ? xv.x : -INFINITY;
        ev.y = k0 + 1 < nc ? xv.y : -INFINITY;
        ev.z = k0 + 2 < nc ? xv.z : -INFINITY;
        ev.w = k0 + 3 < nc ? xv.w : -INFINITY;
    };
    auto jof = [&](int bk, int j0, int c) -> int {
        return contig ? j0 + c : cand_j(bk * 128 + 4 * lane + c);
    };
    // every warp visits its blocks with kUn loads in flight; body(bk, scores[4], j0)
    // Contiguous layouts: every thread prefetches its own float4 of scores (and, when node
    // ids are needed, its union-list entry) kPD - 1 iterations ahead with cp.async into a
    // private slot of a shared-memory ring laid out [slot][thread] (a warp's 32 float4 of one
    // slot are 512 contiguous bytes); it reads back only what it copied, so no barrier is
    // needed.  need_j is a compile-time flag (std::true_type / std::false_type).
    auto stream = [&](auto nj, auto&& body) {
        constexpr bool need_j = decltype(nj)::value;
        const int niter = warp < nblk ? (nblk - warp + nwarps - 1) / nwarps : 0;   // uniform in a warp
        const bool want_u = need_j && !top;
        const int kStep = nwarps * 128;                 // candidates between a thread's iterations
        const int kb0 = warp * 128 + 4 * lane;
        const uint32_t ring = smem_u32(pref + threadIdx.x);
        const uint32_t ringj = smem_u32(prefj + threadIdx.x);
        auto issue = [&](int t) {
            const int k0 = kb0 + t * kStep;
            const bool in = t < niter && k0 < nc;
            const uint32_t sl = (uint32_t)(t & (kPD - 1));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(ring + sl * (NT * 16)),
                         "l"(e + (in ? k0 : 0)), "r"(in ? 16u : 0u)
                         : "memory");
            if (want_u) {
                const int uk = in ? (cs >= 0 ? (k0 >> cs) : k0 / C) : 0;
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(ringj + sl * (NT * 4)),
                             "l"(ul + uk), "r"(in ? 4u : 0u)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
#pragma unroll
        for (int t = 0; t < kPD - 1; ++t) issue(t);
        for (int t = 0; t < niter; ++t) {
            issue(t + kPD - 1);
            asm volatile("cp.async.wait_group %0;" ::"n"(kPD - 1) : "memory");
            const int k0 = kb0 + t * kStep;
            const int sl = t & (kPD - 1);
            float4 ev = pref[sl * NT + threadIdx.x];
            if (k0 + 3 >= nc) {                         // the row's last, partial float4
                ev.x = k0 < nc ? ev.x : -INFINITY;
                ev.y = k0 + 1 < nc ? ev.y : -INFINITY;
                ev.z = k0 + 2 < nc ? ev.z : -INFINITY;
                ev.w = -INFINITY;
            }
            int j0 = -1;
            if constexpr (need_j) {
                if (k0 < nc) {
                    if (top) {
                        j0 = k0;
                    } else {
                        const int pj = prefj[sl * NT + threadIdx.x];
                        j0 = cs >= 0 ? (pj << cs) + (k0 & (C - 1)) : pj * C + (k0 - (k0 / C) * C);
                    }
                }
            }
            body(warp + t * nwarps, ev, j0);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
    };
    auto for_cands = [&](auto nj, auto&& body) {
        if (contig) {
            stream(nj, body);
            return;
        }
        for (int b0 = warp; b0 < nblk; b0 += kUn * nwarps) {
            float4 ev[kUn];
            int j0[kUn];
#pragma unroll
            for (int u = 0; u < kUn; ++u) load(b0 + u * nwarps, ev[u], j0[u], decltype(nj)::value);
#pragma unroll
            for (int u = 0; u < kUn; ++u) {
                const int bk = b0 + u * nwarps;
                if (bk >= nblk) break;
                body(bk, ev[u], j0[u]);
            }
        }
    };
    // kept bits of candidates k0..k0+3 (nibble) into the bitmap: one plain store per
    // 32-candidate word when the warp's 8-lane group covers a whole aligned word (the
    // bitmap starts zeroed), else atomics
    auto put_bits = [&](int bk, uint32_t nib, int j0) {
        if (contig) {
            const int jf = __shfl_sync(kFull, j0, lane & ~7);
            const int jl = __shfl_sync(kFull, j0, lane | 7);
            uint32_t wv = nib << (4 * (lane & 7));
            wv |= __shfl_xor_sync(kFull, wv, 1);
            wv |= __shfl_xor_sync(kFull, wv, 2);
            wv |= __shfl_xor_sync(kFull, wv, 4);
            const bool whole = jf >= 0 && (jf & 31) == 0 && jl == jf + 28;
            if (whole && (lane & 7) == 0 && wv) outw[jf >> 5] = wv;
            if (!whole && nib) atomicOr(outw + (j0 >> 5), nib << (j0 & 31));
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if ((nib >> c) & 1u) {
                    const int j = jof(bk, j0, c);
                    atomicOr(outw + (j >> 5), 1u << (j & 31));
                }
        }
    };

    int bstar = kNB;               // bins < bstar are kept whole
    unsigned long long need = 0;   // mass still needed from the boundary bin
    if (b.p < 1.0f) {
        // pass 1: fixed-point masses into bins of (M - e)
        for (int i = threadIdx.x; i < kNB; i += blockDim.x) {
            hlo[i] = 0u;
            hhi[i] = 0u;
        }
        if (threadIdx.x == 0) s_nkeys = 0;
        __syncthreads();
        if (phase == 2) {
            // sharded cut: the histogram summed over the ranks replaces this rank's own
            for (int i = threadIdx.x; i < kNB; i += blockDim.x) {
                const unsigned long long hv = w.sh_hist[x * kShardBins + i];
                hlo[i] = (uint32_t)hv;
                hhi[i] = (uint32_t)(hv >> 32);
            }
        } else {
            for_cands(std::false_type{}, [&](int bk, const float4 ev4, int j0) {
                const float v[4] = {ev4.x, ev4.y, ev4.z, ev4.w};
                // -inf (off the frontier) gives mass 0 and the last bin: computed without
                // branches, the atomics are predicated
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t lo, hi;
                    sm.mass2(v[c], lo, hi);
                    hist_add(smem_u32(hlo + sm.bin(v[c])), smem_u32(hhi + sm.bin(v[c])), lo, hi);
                }
            });
        }
        __syncthreads();
        if (phase == 1) {
            // sharded cut, first step: this rank's histogram out, to be summed over the ranks
            for (int i = threadIdx.x; i < kNB; i += blockDim.x) w.sh_hist[x * kShardBins + i] = hist(i);
            return;
        }
        // boundary bin b*: cum(bins < b*) < target <= cum(bins <= b*).  Thread t owns the BPT
        // bins from BPT t; one block-wide exclusive scan of the per-thread sums gives Z and
        // each thread's prefix, and the thread whose range holds the target finds b* there.
        constexpr int BPT = kNB / NT;
        static_assert(BPT % 4 == 0, "whole 16-byte groups of bins per thread");
        if (threadIdx.x == 0) {   // only kept if no range holds the target (Z = 0)
            s_bstar = kNB - kNB / 32;
            s_cumb = 0;
        }
        unsigned long long hb[BPT];
#pragma unroll
        for (int v = 0; v < BPT / 4; ++v) {
            const uint4 l4 = reinterpret_cast<const uint4*>(hlo)[threadIdx.x * (BPT / 4) + v];
            const uint4 h4 = reinterpret_cast<const uint4*>(hhi)[threadIdx.x * (BPT / 4) + v];
            hb[4 * v + 0] = ((unsigned long long)h4.x << 32) | l4.x;
            hb[4 * v + 1] = ((unsigned long long)h4.y << 32) | l4.y;
            hb[4 * v + 2] = ((unsigned long long)h4.z << 32) | l4.z;
            hb[4 * v + 3] = ((unsigned long long)h4.w << 32) | l4.w;
        }
        unsigned long long loc = 0;
#pragma unroll
        for (int k = 0; k < BPT; ++k) loc += hb[k];
        unsigned long long Z;
        const unsigned long long excl = block_excl_scan<unsigned long long>(loc, red_u, Z);
        unsigned long long target = (unsigned long long)ceil((double)b.p * (double)Z);
        if (target < 1ull) target = 1ull;
        if (target > Z) target = Z;
        if (excl < target && target <= excl + loc) {
            unsigned long long cum = excl, cumb = excl;
            int bs = BPT * threadIdx.x + BPT - 1;
            bool hit = false;
#pragma unroll
            for (int k = 0; k < BPT; ++k) {
                if (!hit && cum + hb[k] >= target) {
                    hit = true;
                    bs = BPT * threadIdx.x + k;
                    cumb = cum;
                }
                cum += hb[k];
            }
            s_bstar = bs;
            s_cumb = cumb;
        }
        __syncthreads();
        bstar = s_bstar;
        need = target - s_cumb;
    }

    // pass 2: kept bits of the bins above the boundary; boundary-bin candidates collected
    unsigned long long cnt = 0;
    for_cands(std::true_type{}, [&](int bk, const float4 ev4, int j0) {
        const float v[4] = {ev4.x, ev4.y, ev4.z, ev4.w};
        uint32_t nib = 0, col = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const bool ok = v[c] > -INFINITY;
            const int bn = sm.bin(v[c]);
            nib |= (ok && bn < bstar ? 1u : 0u) << c;
            col |= (ok && bn == bstar ? 1u : 0u) << c;
        }
        // boundary-bin candidates: one shared-memory atomic per warp reserves their slots
        if (__any_sync(kFull, col != 0)) {
            const int mine = __popc(col);
            int incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += t;
            }
            unsigned base0 = 0;
            if (lane == 31) base0 = atomicAdd(&s_nkeys, (unsigned)incl);
            base0 = __shfl_sync(kFull, base0, 31);
            unsigned idx = base0 + (unsigned)(incl - mine);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if ((col >> c) & 1u) {
                    if (idx < (unsigned)kCap) keys[idx] = sel_key(v[c], (int)(jof(bk, j0, c) + w.sh_off));
                    ++idx;
                }
        }
        cnt += __popc(nib);
        put_bits(bk, nib, j0);
    });
    cnt = block_sum<unsigned long long>(cnt, red_u);
    if (bstar == kNB) {
        if (threadIdx.x == 0) {
            *kcount = (int32_t)cnt;
            if (phase == 2) {
                w.sh_nkeys[x] = 0;
                w.sh_need[x] = 0;
            }
        }
        return;
    }
    __syncthreads();

    const unsigned nkeys = s_nkeys;
    if (phase == 2) {
        // sharded cut, second step: this rank's boundary-bin keys out, to be gathered from
        // every rank (more than kShardKeys cannot be exchanged: the last step flags it)
        const int nk = (int)min(nkeys, (unsigned)kShardKeys);
        for (int i = threadIdx.x; i < nk; i += blockDim.x) w.sh_keys[x * kShardKeys + i] = keys[i];
        if (threadIdx.x == 0) {
            w.sh_nkeys[x] = (int32_t)nkeys;
            w.sh_need[x] = need;
            *kcount = (int32_t)cnt;
        }
        return;
    }
    if (nkeys <= (unsigned)kCap) {
        // sort the boundary bin by (e desc, j asc) and take the prefix reaching the target
        const int found = sort_prefix(keys, (int)nkeys, need);
        for (int i = threadIdx.x; i <= found; i += blockDim.x) {
            const uint32_t jk = (uint32_t)keys[i];
            atomicOr(outw + (jk >> 5), 1u << (jk & 31));
        }
        if (threadIdx.x == 0) s_found = found + 1;
    } else {
        // rare: too many candidates in one bin - bisection on the exact key order, then a pass
        unsigned long long klo = ~0ull, khi = 0ull;
        for_cands(std::true_type{}, [&](int bk, const float4 ev4, int j0) {
        const float v[4] = {ev4.x, ev4.y, ev4.z, ev4.w};
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (v[c] > -INFINITY && sm.bin(v[c]) == bstar) {
                    const unsigned long long kk = sel_key(v[c], jof(bk, j0, c));
                    klo = kk < klo ? kk : klo;
                    khi = kk > khi ? kk : khi;
                }
        });
        unsigned long long lo = block_min_t<unsigned long long>(klo, red_u);
        unsigned long long hi = block_max_t<unsigned long long>(khi, red_u);
        int iters = 0;
        while (lo < hi && iters < 70) {
            const unsigned long long mid = lo + (hi - lo) / 2;
            unsigned long long acc = 0;
            for_cands(std::true_type{}, [&](int bk, const float4 ev4, int j0) {
        const float v[4] = {ev4.x, ev4.y, ev4.z, ev4.w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (v[c] > -INFINITY && sm.bin(v[c]) == bstar && sel_key(v[c], jof(bk, j0, c)) <= mid)
                        acc += sm.mass(v[c]);
            });
            acc = block_sum<unsigned long long>(acc, red_u);
            if (acc >= need) hi = mid;
            else lo = mid + 1;
            ++iters;
        }
        if (threadIdx.x == 0 && iters >= 70) atomicOr(w.status, kStatusSelectFallbackLimit);
        unsigned long long extra = 0;
        for_cands(std::true_type{}, [&](int bk, const float4 ev4, int j0) {
        const float v[4] = {ev4.x, ev4.y, ev4.z, ev4.w};
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (v[c] > -INFINITY && sm.bin(v[c]) == bstar) {
                    const int j = jof(bk, j0, c);
                    if (sel_key(v[c], j) <= lo) {
                        atomicOr(outw + (j >> 5), 1u << (j & 31));
                        ++extra;
                    }
                }
        });
        extra = block_sum<unsigned long long>(extra, red_u);
        if (threadIdx.x == 0) s_found = (int)extra;
    }
    __syncthreads();
    if (threadIdx.x == 0) *kcount = (int32_t)(cnt + (unsigned long long)s_found);
}

int score_blocks_x(int lane_blocks, int groups) {
    const int target = sm_count() * 8;
    int nb = target / max(1, lane_blocks * groups);
    return nb < 1 ? 1 : (nb > 65535 ? 65535 : nb);
}

}  // namespace

cudaError_t launch_union(const Batch& b, const Work& w, int it, int mode, cudaStream_t st) {
    ProfScope ps_("k_union", st);
    cudaError_t e = cudaMemsetAsync(w.uword, 0, (size_t)b.n_groups * w.uw * 4, st);
    if (e != cudaSuccess) return e;
    const int lanes_per_block = 64;
    dim3 grid((unsigned)((w.uw + 255) / 256), (b.n_gl + lanes_per_block - 1) / lanes_per_block, b.n_groups);
    k_union_or<<<grid, 256, 0, st>>>(b, w, it, mode, lanes_per_block);
    const unsigned chunks = (unsigned)std::max<int64_t>(1, (w.uw + kCompactWords - 1) / kCompactWords);
    k_union_compact<<<dim3(chunks, b.n_groups), kCompactThreads, 0, st>>>(b, w, it, mode);
    return cudaGetLastError();
}

cudaError_t launch_score(const Batch& b, const Work& w, int it, float scale, cudaStream_t st) {
    const bool tc = b.all_r16 && w.tmaps && b.fmt != kFmtFp4 &&
                    (b.score_path == 2 || b.score_path == 0);
    if (tc) return launch_score_tc(b, w, it, scale, st);
    if (b.all_r16 && b.n_gl <= kFewLanes && b.d == 128) {
        // one wave: 2 blocks of 8 warps per SM, shared by the groups (d = 128, the geometry
        // the few-lane kernel is validated on; d = 64 takes k_score)
        const int bx = std::max(1, 2 * sm_count() / std::max(1, b.n_groups));
        ProfScope ps_("k_score", st);
        if (b.fmt == kFmtBf16)
            k_score_few<128, kFmtBf16><<<dim3(bx, 1, b.n_groups), 256, 0, st>>>(b, w, it, scale);
        else if (b.fmt == kFmtFp4)
            k_score_few<128, kFmtFp4><<<dim3(bx, 1, b.n_groups), 256, 0, st>>>(b, w, it, scale);
        else
            k_score_few<128, kFmtF16x2><<<dim3(bx, 1, b.n_groups), 256, 0, st>>>(b, w, it, scale);
        return cudaGetLastError();
    }
    const int WB = min(8, (b.n_gl + 7) / 8);
    const int lane_blocks = (b.n_gl + 8 * WB - 1) / (8 * WB);
    dim3 grid(score_blocks_x(lane_blocks, b.n_groups), lane_blocks, b.n_groups);
    ProfScope ps_("k_score", st);
    if (b.d == 128) {
        if (b.fmt == kFmtBf16) k_score<128, kFmtBf16><<<grid, 256, 0, st>>>(b, w, it, scale);
        else if (b.fmt == kFmtFp4) k_score<128, kFmtFp4><<<grid, 256, 0, st>>>(b, w, it, scale);
        else k_score<128, kFmtF16x2><<<grid, 256, 0, st>>>(b, w, it, scale);
    } else {
        if (b.fmt == kFmtBf16) k_score<64, kFmtBf16><<<grid, 256, 0, st>>>(b, w, it, scale);
        else if (b.fmt == kFmtFp4) k_score<64, kFmtFp4><<<grid, 256, 0, st>>>(b, w, it, scale);
        else k_score<64, kFmtF16x2><<<grid, 256, 0, st>>>(b, w, it, scale);
    }
    return cudaGetLastError();
}

cudaError_t launch_select(const Batch& b, const Work& w, int it, int64_t max_cands, cudaStream_t st) {
    ProfScope ps_("k_select", st);
    // Lanes with few candidates (upper levels) are latency-bound: small blocks, more per SM.
    auto go = [&](auto kern, int nt) {
        const size_t smem = (size_t)kNB * 8 + (size_t)kCap * 8 + (size_t)nt * kPD * (16 + 4);
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<b.n_lanes, nt, smem, st>>>(b, w, it);
    };
    if (max_cands <= kSelSmallCands)
        go(k_select<kSelThreadsSmall>, kSelThreadsSmall);
    else
        go(k_select<kSelThreads>, kSelThreads);
    return cudaGetLastError();
}

}  // namespace zha
