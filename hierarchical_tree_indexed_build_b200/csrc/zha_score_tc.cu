// zha_score_tc.cu - plane-estimate scoring on the 5th-generation tensor cores (tcgen05).
//
// Same quantity as k_score (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的:
// 取这些平面的最大值; wqu.guru, section "Building the tree"): for every lane of a
// (sequence, KV head) group and every candidate node j on the lane's frontier,
//     e_j = max_r ( s q.m_r(j) + b_r(j) ),
// and -inf for candidates off the lane's frontier (children of nodes other lanes kept).
// When a group holds many lanes (query tokens x GQA heads) this is a dense contraction
// D[lane][(node, r)] = sum_k Q[lane][k] m_r(j)[k], run here as tcgen05.mma kind::f16 with
// M = 128 lanes, N = 8 nodes x 16 planes, K = d, f32 accumulators in tensor memory.
//
// Precision: Q is bf16, which fp16 holds exactly for magnitudes in [2^-17, 65504).  The
// f32 summary m is split into two fp16 terms m = hi + lo (lo the fp16 rounding of m - hi),
// so two MMA passes accumulate Q.m with an error of at most 2^-22 |m| + 2^-25 per
// element: float32-grade scores.  An entry of Q or m of magnitude >= 65504 does not fit;
// the kernel then sets kStatusRange (the CUDA-core scorer has no such limit).
//
// Pipeline (one CTA per SM, persistent over its node tiles; LT = 1 or 2 lane tiles of 128
// lanes per CTA share every node tile, so one read of a node serves 128 LT lanes):
//   warps 0-7   producers: load a node tile (f32, one tile in flight in registers), split it
//               into the two fp16 planes and store them in a 128-byte-swizzled K-major
//               shared-memory stage (2 stages), with the tile's b values, node ids and the
//               frontier-membership words of the CTA's lanes;
//   warps 8..   epilogue, 4 per lane tile: tensor memory -> max over planes + b -> scores;
//               lane 0 of warp 8 also issues the MMAs into one of two TMEM accumulators per
//               lane tile (the next tile's as soon as its operands are staged).
// Shared-memory operand layout: per K block of 64 fp16, rows are 128 bytes apart, the
// 16-byte chunk c of row r sits at chunk c ^ (r % 8), 8-row groups 1024 bytes apart.
//
// Frontier membership comes from k_member: for every union parent u of the level above
// and every 32 lanes of the group, one word whose bit t says whether lane 32 w + t kept u
// (the lanes' kept bitmaps transposed), so the scorer reads membership with the node data.
#include <cuda_fp16.h>
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

size_t score_tc_smem_lt(int d, int lt);

namespace {

constexpr int kTileM = 128;          // lanes per tile (MMA M)
constexpr int kTileN = 128;          // rows (node, plane) per tile (MMA N)
constexpr int kR = 16;               // planes per node on this path
constexpr int kNodes = kTileN / kR;  // nodes per tile
constexpr int kProducers = 256;      // warps 0-7
constexpr int kMmaWarp = kProducers / 32;   // first epilogue warp: issues MMAs, owns TMEM
constexpr int kChunk = kProducers / kNodes;   // tiles whose node ids are staged at once
constexpr int kPlanes = 2;           // fp16 terms of m
constexpr float kHalfMax = 65504.0f; // largest finite fp16
constexpr uint64_t kWaitNs = 2000000000ull;   // bound on any wait for the tensor pipeline

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major, 128B-swizzle UMMA shared-memory descriptor (sm_100 format, version 1).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);      // start address
    d |= (uint64_t)1 << 16;                       // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: 8-row groups
    d |= (uint64_t)1 << 46;                       // descriptor version
    d |= (uint64_t)2 << 61;                       // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16 with fp16 A/B, f32 accumulate, both K-major, M x N.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(a), "l"(b), "r"(kIdesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// Waits for the mbarrier phase with the given parity; gives up after about 2 s of wall time.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
        uint64_t t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > kWaitNs) return false;
    }
}

// Non-blocking probe: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t mbar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Byte offset of element d (16-bit) of row `row` in a K-major tile of 128-row, 128-byte blocks.
__device__ __forceinline__ uint32_t swz16(int row, int d) {
    const int kb = d >> 6, c = (d & 63) >> 3;
    return (uint32_t)(kb * (128 * 128) + row * 128 + ((c ^ (row & 7)) << 4) + (d & 7) * 2);
}

// m = hi + lo, hi the fp16 rounding of m and lo that of m - hi; two elements per word.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Lanes' kept bits of the level above, transposed: memb[grp][u][w] bit t = lane 32 w + t
// kept union parent u.  Grid (parent chunks, lane words, groups); a warp covers 32 parents.
__global__ void __launch_bounds__(256) k_member(Batch b, Work w, int it) {
    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int lev = sq.L - it;
    if (lev < 1 || lev == sq.L) return;           // top level: no parents
    const int pl = lev + 1;
    const int nu = w.ucount[grp];
    const int lw = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int y = lw * 32 + lane;
    const bool ok = y < b.n_gl;
    const uint32_t* kb = w.kept[pl] + lane_of(b, s, g, ok ? y : 0) * w.W[pl];
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    uint32_t* out = w.memb + (int64_t)grp * w.ms * w.mwords + lw;
    for (int c = blockIdx.x * 8 + warp; c * 32 < nu; c += gridDim.x * 8) {
        const int u0 = c * 32, n = min(32, nu - u0);
        const int pmy = lane < n ? __ldg(ul + u0 + lane) : -1;
        const int p0 = __shfl_sync(0xffffffffu, pmy, 0);
        const int pn = __shfl_sync(0xffffffffu, pmy, n - 1);
        uint32_t mine = 0;
        if (n == 32 && (p0 & 31) == 0 && pn == p0 + 31) {
            // 32 consecutive parents: one bitmap word per lane, transposed by ballots
            const uint32_t word = ok ? __ldg(kb + (p0 >> 5)) : 0u;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const uint32_t r = __ballot_sync(0xffffffffu, (word >> t) & 1u);
                if (lane == t) mine = r;
            }
        } else {
            for (int t = 0; t < n; ++t) {
                const int pt = __shfl_sync(0xffffffffu, pmy, t);
                const uint32_t bit = ok ? (__ldg(kb + (pt >> 5)) >> (pt & 31)) & 1u : 0u;
                const uint32_t r = __ballot_sync(0xffffffffu, bit);
                if (lane == t) mine = r;
            }
        }
        if (lane < n) out[(int64_t)(u0 + lane) * w.mwords] = mine;
    }
}

template <int D, int LT>
__global__ void __launch_bounds__(kProducers + 128 * LT, 1) k_score_tc(Batch b, Work w, int it, float scale) {
    constexpr int kThreads = kProducers + 128 * LT;
    constexpr int kEpilogue = 128 * LT;
    constexpr int kLW = 4 * LT;                       // 32-lane membership words per CTA
    constexpr int KB = D / 64;                        // 128-byte K blocks of 16-bit elements
    constexpr int A_BYTES = KB * kTileM * 128;        // one lane tile
    constexpr int P_BYTES = KB * kTileN * 128;        // one fp16 plane of one stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = base;                                             // [LT][A_BYTES]
    unsigned char* sB0 = base + LT * A_BYTES;                             // [2 stages][2 planes][P_BYTES]
    float* sBv = reinterpret_cast<float*>(sB0 + 2 * kPlanes * P_BYTES);   // [2][kTileN] b values
    uint32_t* sMask = reinterpret_cast<uint32_t*>(sBv + 2 * kTileN);     // [2][kLW][kNodes] membership
    int32_t* sJ = reinterpret_cast<int32_t*>(sMask + 2 * kLW * kNodes);  // [2][kNodes] node ids (-1: none)
    int32_t* sNode = sJ + 2 * kNodes;                                     // [2][kChunk * kNodes] staged ids
    __shared__ __align__(8) uint64_t bar_full[2], bar_acc_full[2], bar_acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    volatile int& abort_sh = abort_flag;              // set by any role whose wait gave up

    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int lev = sq.L - it;
    if (lev < 1) return;
    const bool top = (lev == sq.L);
    const int C = sq.C;
    const int nc = (int)(top ? sq.T : (int64_t)w.ucount[grp] * C);   // < 2^31: level-1 nodes <= 2^24
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        atomicAdd(&w.ctr[kCtrUnionNodes + lev], (unsigned long long)nc);
    const int ntiles = (nc + kNodes - 1) / kNodes;
    if ((int)blockIdx.x >= ntiles) return;          // whole block leaves before any barrier
    const int nt = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;   // tiles of this block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y0 = blockIdx.y * (kTileM * LT);
    const uint32_t ncols = 2 * kTileN * LT;           // two accumulators per lane tile

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bar_full[i]), kProducers);
            mbar_init(smem_u32(&bar_acc_full[i]), 1);
            mbar_init(smem_u32(&bar_acc_empty[i]), kEpilogue);
        }
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    // A: the CTA's query rows (bf16 -> fp16, exact in range), zero rows past the group's lanes.
    float amax = 0.0f;
    for (int i = tid; i < LT * kTileM * (D / 8); i += kThreads) {
        const int row = i / (D / 8), c16 = i % (D / 8);
        const int y = y0 + row;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (y < b.n_gl) v = __ldg(reinterpret_cast<const uint4*>(b.Q + lane_of(b, s, g, y) * D) + c16);
        uint32_t hv[4];
        const uint32_t* bv = &v.x;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(bv + t));
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            const __half2 h = __floats2half2_rn(f.x, f.y);
            hv[t] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(sA + (row / kTileM) * A_BYTES + swz16(row % kTileM, c16 * 8)) =
            make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    if (!(amax < kHalfMax)) atomicOr(w.status, kStatusRange);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_sh;

    const int64_t ns = sq.ns;
    const float* recb = sq.rec[lev] + (int64_t)g * sq.cap[lev] * ns;
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    const uint32_t* memb = w.memb + (int64_t)grp * w.ms * w.mwords + (int64_t)blockIdx.y * kLW;

    if (warp < kProducers / 32) {
        // ---------------- producers
        constexpr int kRowStep = kProducers / (D / 4);
        constexpr int kU = kTileN / kRowStep;         // float4 per thread per tile
        const int c4 = tid % (D / 4);
        const int row0 = tid / (D / 4);
        float mmax = 0.0f;                            // largest |m| this thread split
        const int lane_words = (b.n_gl + 31) / 32;
        // candidate k of the group -> node index (or -1 past the end)
        auto node_of = [&](int k) -> int {
            if (k >= nc) return -1;
            if (top) return k;
            const uint32_t pk = (uint32_t)k / (uint32_t)C;
            return __ldg(ul + pk) * C + (k - (int)pk * C);
        };
        // Node ids of chunk c (tiles [c kChunk, (c+1) kChunk) of this block) into sNode[c & 1]:
        // one independent load per producer thread, so no tile waits on a dependent load.
        auto fill_chunk = [&](int c) {
            const int i = c * kChunk + tid / kNodes;
            int j = -1;
            if (i < nt) j = node_of((blockIdx.x + i * gridDim.x) * kNodes + tid % kNodes);
            sNode[(c & 1) * kProducers + tid] = j;
        };
        auto node_at = [&](int i, int nl) -> int {
            return sNode[((i / kChunk) & 1) * kProducers + (i % kChunk) * kNodes + nl];
        };
        float4 pre[kU];
        float preb = 0.f;
        int prej = -1;
        uint32_t prem = 0;
        auto prefetch = [&](int i) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int row = row0 + u * kRowStep;
                const int j = node_at(i, row / kR);
                pre[u] = j >= 0 ? __ldg(reinterpret_cast<const float4*>(recb + (int64_t)j * ns + (row % kR) * D) + c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (tid < kTileN) {
                prej = node_at(i, tid / kR);
                preb = prej >= 0 ? __ldg(recb + (int64_t)prej * ns + kR * D + tid % kR) : 0.0f;
            }
            if (tid < kLW * kNodes) {
                // membership word (node tid / kLW, lane word tid % kLW) of tile i
                const int k = (blockIdx.x + i * gridDim.x) * kNodes + tid / kLW;
                const bool wok = (int)blockIdx.y * kLW + tid % kLW < lane_words;   // words past the group's lanes: 0
                prem = (k >= nc || !wok) ? 0u : top ? 0xffffffffu : __ldg(memb + (int64_t)(k / C) * w.mwords + tid % kLW);
            }
        };
        fill_chunk(0);
        fill_chunk(1);
        asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");
        prefetch(0);
        for (int i = 0; i < nt; ++i) {
            const int st = i & 1;
            // stage st (and its metadata) is free once the epilogue of tile i-2 is done.
            // After an abort the producers keep stepping without waiting, so that all of them
            // reach the same named barriers.
            if (i >= 2 && !abort_sh && !mbar_wait(smem_u32(&bar_acc_empty[st]), (uint32_t)(((i >> 1) - 1) & 1))) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            unsigned char* pl = sB0 + (size_t)(kPlanes * st) * P_BYTES;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int row = row0 + u * kRowStep;
                const float4 m = pre[u];
                mmax = fmaxf(mmax, fmaxf(fmaxf(fabsf(m.x), fabsf(m.y)), fmaxf(fabsf(m.z), fabsf(m.w))));
                uint32_t h0, l0, h1, l1;
                split2(m.x, m.y, h0, l0);
                split2(m.z, m.w, h1, l1);
                const uint32_t off = swz16(row, c4 * 4);
                *reinterpret_cast<uint2*>(pl + off) = make_uint2(h0, h1);
                *reinterpret_cast<uint2*>(pl + P_BYTES + off) = make_uint2(l0, l1);
            }
            if (tid < kTileN) {
                sBv[st * kTileN + tid] = preb;
                if (tid % kR == 0) sJ[st * kNodes + tid / kR] = prej;
            }
            if (tid < kLW * kNodes) sMask[st * kLW * kNodes + (tid % kLW) * kNodes + tid / kLW] = prem;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(smem_u32(&bar_full[st]));
            // tile i + 1 may open the next chunk: stage its node ids one chunk ahead
            if ((i + 1) % kChunk == 0 && i + 1 < nt) {
                asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");   // old ids of that buffer consumed
                fill_chunk((i + 1) / kChunk + 1);
            }
            if ((i + 1) % kChunk == 0)
                asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");   // new ids visible
            if (i + 1 < nt) prefetch(i + 1);
        }
        if (!(mmax < kHalfMax)) atomicOr(w.status, kStatusRange);
    } else {
        // ---------------- epilogue: scores of tile i from accumulator i % 2 of each lane tile.
        // Lane 0 of the first epilogue warp also issues the MMAs: tile i+1's before this
        // warp drains tile i when its operands are already staged, else right after the
        // drain, so the epilogue never waits on the producers while an accumulator is full.
        const int ew = warp - kProducers / 32;
        const int lt = ew >> 2, quad = warp & 3;      // TMEM lane quarter = warp % 4
        const int row = lt * kTileM + quad * 32 + lane;
        const int y = y0 + row;
        const bool ok = y < b.n_gl;
        const int64_t x = lane_of(b, s, g, ok ? y : 0);
        float* ex = w.e + x * w.es;
        float fmax = -INFINITY;
        int fcnt = 0;
        const bool issuer = warp == kMmaWarp && lane == 0;
        auto issue = [&](int i) {
            const int st = i & 1;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t pl0 = smem_u32(sB0 + (size_t)(kPlanes * st) * P_BYTES);
            // descriptors advance by the operand offset in 16-byte units (start-address field);
            // loops kept rolled so the compiler does not hold every descriptor in registers
#pragma unroll 1
            for (int t = 0; t < LT; ++t) {
                const uint32_t d = tmem + (uint32_t)((t * 2 + st) * kTileN);
                const uint64_t da = umma_desc(smem_u32(sA + t * A_BYTES));
                const uint64_t db = umma_desc(pl0);
#pragma unroll 1
                for (int pk = 0; pk < kPlanes * KB; ++pk) {
                    const int pass = pk / KB, kb = pk % KB;
                    const uint64_t a1 = da + (uint64_t)((kb * (kTileM * 128)) >> 4);
                    const uint64_t b1 = db + (uint64_t)((pass * P_BYTES + kb * (kTileN * 128)) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(d, a1 + (uint64_t)(kk * 2), b1 + (uint64_t)(kk * 2), (pk | kk) ? 1u : 0u);
                }
            }
            mma_commit(smem_u32(&bar_acc_full[st]));
        };
        // operands of tile i staged and its accumulators drained (by tile i-2's epilogue)
        auto ready = [&](int i) -> bool {
            const int st = i & 1;
            if (!mbar_test(smem_u32(&bar_full[st]), (uint32_t)((i >> 1) & 1))) return false;
            return i < 2 || mbar_test(smem_u32(&bar_acc_empty[st]), (uint32_t)(((i >> 1) - 1) & 1));
        };
        auto issue_blocking = [&](int i) {
            const int st = i & 1;
            bool okw = mbar_wait(smem_u32(&bar_full[st]), (uint32_t)((i >> 1) & 1));
            if (okw && i >= 2) okw = mbar_wait(smem_u32(&bar_acc_empty[st]), (uint32_t)(((i >> 1) - 1) & 1));
            if (!okw) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (!abort_sh) issue(i);
        };
        if (issuer) issue_blocking(0);
        for (int i = 0; i < nt; ++i) {
            bool issued_next = false;
            if (issuer && i + 1 < nt && !abort_sh && ready(i + 1)) {
                issue(i + 1);
                issued_next = true;
            }
            __syncwarp();
            const int st = i & 1;
            if (!mbar_wait(smem_u32(&bar_acc_full[st]), (uint32_t)((i >> 1) & 1))) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (__any_sync(0xffffffffu, abort_sh != 0)) break;   // warp-uniform: tcgen05.ld below is collective
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // the stage's metadata stays valid until this epilogue releases it: copy it out
            int jv[kNodes];
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) jv[nl] = sJ[st * kNodes + nl];
            uint32_t member = 0;
            {
                const uint4* mk = reinterpret_cast<const uint4*>(sMask + st * kLW * kNodes + (row >> 5) * kNodes);
                const uint4 m0 = mk[0], m1 = mk[1];
                const uint32_t mws[kNodes] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
                for (int nl = 0; nl < kNodes; ++nl) member |= ((mws[nl] >> lane) & 1u) << nl;
            }
            const float4* bv4 = reinterpret_cast<const float4*>(sBv + st * kTileN);
            float best[kNodes];
#pragma unroll
            for (int pr = 0; pr < kNodes / 2; ++pr) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)((lt * 2 + st) * kTileN + pr * 2 * kR), v);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float bb = -INFINITY;
#pragma unroll
                    for (int r4 = 0; r4 < kR / 4; ++r4) {
                        const float4 bq = bv4[(pr * 2 + h) * (kR / 4) + r4];
                        bb = fmaxf(bb, fmaf(scale, v[h * kR + 4 * r4 + 0], bq.x));
                        bb = fmaxf(bb, fmaf(scale, v[h * kR + 4 * r4 + 1], bq.y));
                        bb = fmaxf(bb, fmaf(scale, v[h * kR + 4 * r4 + 2], bq.z));
                        bb = fmaxf(bb, fmaf(scale, v[h * kR + 4 * r4 + 3], bq.w));
                    }
                    best[pr * 2 + h] = bb;
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(smem_u32(&bar_acc_empty[st]));
            if (issuer && i + 1 < nt && !issued_next) issue_blocking(i + 1);
            // scores out: -inf off the frontier; 16-byte stores where 4 nodes are consecutive
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) {
                if ((member >> nl) & 1u) {
                    fmax = fmaxf(fmax, best[nl]);
                    ++fcnt;
                } else {
                    best[nl] = -INFINITY;
                }
            }
            if (ok) {
#pragma unroll
                for (int q4 = 0; q4 < kNodes / 4; ++q4) {
                    const int j0 = jv[4 * q4], j3 = jv[4 * q4 + 3];
                    if (j0 >= 0 && (j0 & 3) == 0 && j3 == j0 + 3) {
                        *reinterpret_cast<float4*>(ex + j0) =
                            make_float4(best[4 * q4], best[4 * q4 + 1], best[4 * q4 + 2], best[4 * q4 + 3]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if (jv[4 * q4 + c] >= 0) ex[jv[4 * q4 + c]] = best[4 * q4 + c];
                    }
                }
            }
        }
        if (ok && fcnt > 0) {
            atomicMax(w.lane_max + (int64_t)lev * w.lanes_cap + x, ord_bits(fmax));
            atomicAdd(w.lane_cnt + (int64_t)lev * w.lanes_cap + x, fcnt);
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
}

template <int D, int LT>
cudaError_t launch_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st, int pairs) {
    int nb = 148 / max(1, pairs * b.n_groups);
    nb = nb < 1 ? 1 : nb;
    dim3 grid(nb, pairs, b.n_groups);
    const size_t smem = score_tc_smem_lt(D, LT);
    cudaFuncSetAttribute(k_score_tc<D, LT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_score_tc<D, LT><<<grid, kProducers + 128 * LT, smem, st>>>(b, w, it, scale);
    return cudaGetLastError();
}

}  // namespace

size_t score_tc_smem_lt(int d, int lt) {
    return (size_t)(d / 64) * 128 * 128 * (lt + 2 * kPlanes) + 2 * kTileN * 4 + 2 * 4 * lt * kNodes * 4 +
           2 * kNodes * 4 + 2 * kProducers * 4 + 1024;
}

size_t score_tc_smem(int d) { return score_tc_smem_lt(d, 2); }

cudaError_t launch_score_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st) {
    ProfScope ps_("k_score_tc", st);
    if (it > 0) {
        // membership words of the group's union parents (the level above the scored one)
        const int lw = (b.n_gl + 31) / 32;
        int nbm = (int)((w.ms + 255) / 256);
        nbm = nbm < 1 ? 1 : (nbm > 148 ? 148 : nbm);
        k_member<<<dim3(nbm, lw, b.n_groups), 256, 0, st>>>(b, w, it);
    }
    const int lane_tiles = (b.n_gl + kTileM - 1) / kTileM;
    if (lane_tiles >= 2) {
        const int pairs = (lane_tiles + 1) / 2;
        return b.d == 128 ? launch_tc<128, 2>(b, w, it, scale, st, pairs) : launch_tc<64, 2>(b, w, it, scale, st, pairs);
    }
    return b.d == 128 ? launch_tc<128, 1>(b, w, it, scale, st, 1) : launch_tc<64, 1>(b, w, it, scale, st, 1);
}

}  // namespace zha
