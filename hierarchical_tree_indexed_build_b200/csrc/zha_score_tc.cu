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
// Pipeline (one CTA per SM, persistent over its node tiles):
//   warps 0-7   producers: load a node tile (f32), split into the two fp16 planes, store
//               them in a 128-byte-swizzled K-major shared-memory stage (2 stages);
//   warps 8-11  epilogue: tensor memory -> max over planes + b -> scores; lane 0 of warp 8
//               also issues the MMAs of the next tile into the other TMEM accumulator.
// Shared-memory operand layout: per K block of 64 bf16, rows are 128 bytes apart, the
// 16-byte chunk c of row r sits at chunk c ^ (r % 8), 8-row groups 1024 bytes apart.
#include <cuda_fp16.h>
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr int kTileM = 128;          // lanes per tile (MMA M)
constexpr int kTileN = 128;          // rows (node, plane) per tile (MMA N)
constexpr int kR = 16;               // planes per node on this path
constexpr int kNodes = kTileN / kR;  // nodes per tile
constexpr int kProducers = 256;      // warps 0-7
constexpr int kEpilogue = 128;       // warps 8-11
constexpr int kThreads = kProducers + kEpilogue;
constexpr int kMmaWarp = kProducers / 32;   // first epilogue warp: issues MMAs, owns TMEM
constexpr int kRing = 2;             // node tiles whose loads each producer keeps in flight
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

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1) k_score_tc(Batch b, Work w, int it, float scale) {
    constexpr int KB = D / 64;                        // 128-byte K blocks of 16-bit elements
    constexpr int A_BYTES = KB * kTileM * 128;
    constexpr int P_BYTES = KB * kTileN * 128;        // one fp16 plane of one stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = base;
    unsigned char* sB0 = base + A_BYTES;                                  // [2 stages][2 planes][P_BYTES]
    float* sBv = reinterpret_cast<float*>(sB0 + 2 * kPlanes * P_BYTES);   // [2][kTileN] b values
    int64_t* sJ = reinterpret_cast<int64_t*>(sBv + 2 * kTileN);          // [2][kNodes] node ids (-1: none)
    int32_t* sNode = reinterpret_cast<int32_t*>(sJ + 2 * kNodes);        // [2][kChunk * kNodes] staged ids
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
    const int64_t nc = top ? sq.T : (int64_t)w.ucount[grp] * C;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        atomicAdd(&w.ctr[kCtrUnionNodes + lev], (unsigned long long)nc);
    const int64_t ntiles = (nc + kNodes - 1) / kNodes;
    if ((int64_t)blockIdx.x >= ntiles) return;      // whole block leaves before any barrier
    const int64_t nt = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;   // tiles of this block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y0 = blockIdx.y * kTileM;

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(2 * kTileN));
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
    // A: the tile's query rows (bf16 -> fp16, exact in range), zero rows past the group's lanes.
    float amax = 0.0f;
    for (int i = tid; i < kTileM * (D / 8); i += kThreads) {
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
        *reinterpret_cast<uint4*>(sA + swz16(row, c16 * 8)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
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
    auto node_of = [&](int64_t t, int nl) -> int64_t {
        const int64_t k = t * kNodes + nl;
        if (k >= nc) return -1;
        return top ? k : (int64_t)__ldg(ul + k / C) * C + k % C;
    };

    if (warp < kProducers / 32) {
        // ---------------- producers
        constexpr int kRowStep = kProducers / (D / 4);
        constexpr int kU = kTileN / kRowStep;         // float4 per thread per tile
        const int c4 = tid % (D / 4);
        const int row0 = tid / (D / 4);
        float mmax = 0.0f;   // largest |m| this thread split
        // Node ids of chunk c (tiles [c kChunk, (c+1) kChunk) of this block) into sNode[c & 1]:
        // one independent load per producer thread, so no tile waits on a dependent load.
        auto fill_chunk = [&](int64_t c) {
            const int64_t i = c * kChunk + tid / kNodes;
            int32_t j = -1;
            if (i < nt) j = (int32_t)node_of(blockIdx.x + i * gridDim.x, tid % kNodes);
            sNode[(c & 1) * kProducers + tid] = j;
        };
        auto node_at = [&](int64_t i, int nl) -> int64_t {
            return sNode[((i / kChunk) & 1) * kProducers + (i % kChunk) * kNodes + nl];
        };
        auto prefetch = [&](int64_t i, float4 (&pre)[kU], float& preb, int64_t& prej) {
            if (i >= nt) return;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int row = row0 + u * kRowStep;
                const int64_t j = node_at(i, row / kR);
                pre[u] = j >= 0 ? __ldg(reinterpret_cast<const float4*>(recb + j * ns + (int64_t)(row % kR) * D) + c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (tid < kTileN) {
                prej = node_at(i, tid / kR);
                preb = prej >= 0 ? __ldg(recb + prej * ns + (int64_t)kR * D + tid % kR) : 0.0f;
            }
        };
        // stage tile i from its ring slot, then refill the slot with tile i + kRing
        auto step = [&](int64_t i, float4 (&pre)[kU], float& preb, int64_t& prej) -> bool {
            if (i >= nt) return false;
            const int st = (int)(i & 1);
            // stage st (and its b / node ids) is free once the epilogue of tile i-2 is done.
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
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(smem_u32(&bar_full[st]));
            // tile i + kRing may open the next chunk: stage its node ids one chunk ahead
            if ((i + kRing) % kChunk == 0 && i + kRing < nt) {
                asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");   // old ids of that buffer consumed
                fill_chunk((i + kRing) / kChunk + 1);
            }
            if ((i + kRing) % kChunk == 0)
                asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");   // new ids visible
            prefetch(i + kRing, pre, preb, prej);
            return true;
        };
        fill_chunk(0);
        fill_chunk(1);
        asm volatile("bar.sync 1, %0;" ::"n"(kProducers) : "memory");
        float4 p0[kU], p1[kU];
        float b0 = 0.f, b1 = 0.f;
        int64_t j0 = -1, j1 = -1;
        prefetch(0, p0, b0, j0);
        prefetch(1, p1, b1, j1);
        for (int64_t i = 0; i < nt; i += kRing) {
            if (!step(i, p0, b0, j0)) break;
            if (!step(i + 1, p1, b1, j1)) break;
        }
        if (!(mmax < kHalfMax)) atomicOr(w.status, kStatusRange);
    } else {
        // ---------------- epilogue: scores of tile i from accumulator i % 2.  Lane 0 of the
        // first epilogue warp issues tile i+1's MMAs before this warp drains tile i.
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int y = y0 + row;
        const bool ok = y < b.n_gl;
        const int64_t x = lane_of(b, s, g, ok ? y : 0);
        float* ex = w.e + x * w.es;
        // the lane's kept set one level up decides which candidates are on its frontier
        const uint32_t* Pb = top ? nullptr : w.kept[lev + 1] + x * w.W[lev + 1];
        float fmax = -INFINITY;
        int fcnt = 0;
        const bool issuer = warp == kMmaWarp && lane == 0;
        const uint32_t a0 = smem_u32(sA);
        auto issue = [&](int64_t i) {
            const int st = (int)(i & 1);
            bool okw = mbar_wait(smem_u32(&bar_full[st]), (uint32_t)((i >> 1) & 1));
            if (okw && i >= 2) okw = mbar_wait(smem_u32(&bar_acc_empty[st]), (uint32_t)(((i >> 1) - 1) & 1));
            if (!okw) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (abort_sh) return;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t d = tmem + (uint32_t)(st * kTileN);
            const uint32_t pl0 = smem_u32(sB0 + (size_t)(kPlanes * st) * P_BYTES);
#pragma unroll
            for (int pass = 0; pass < kPlanes; ++pass)
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(d, umma_desc(a0 + kb * (kTileM * 128) + kk * 32),
                                 umma_desc(pl0 + pass * P_BYTES + kb * (kTileN * 128) + kk * 32),
                                 (pass | kb | kk) ? 1u : 0u);
            mma_commit(smem_u32(&bar_acc_full[st]));
        };
        if (issuer) issue(0);
        for (int64_t i = 0; i < nt; ++i) {
            if (issuer && i + 1 < nt) issue(i + 1);
            __syncwarp();
            const int st = (int)(i & 1);
            if (!mbar_wait(smem_u32(&bar_acc_full[st]), (uint32_t)((i >> 1) & 1))) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (__any_sync(0xffffffffu, abort_sh != 0)) break;   // warp-uniform: tcgen05.ld below is collective
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            uint32_t member = 0;
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) {
                const int64_t j = sJ[st * kNodes + nl];
                bool mb = j >= 0;
                if (mb && !top) {
                    const int64_t pj = j / C;
                    mb = (__ldg(Pb + (pj >> 5)) >> (pj & 31)) & 1u;
                }
                member |= (mb ? 1u : 0u) << nl;
            }
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) {
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(st * kTileN + nl * kR), v);
                float best = -INFINITY;
#pragma unroll
                for (int r = 0; r < kR; ++r) best = fmaxf(best, fmaf(scale, v[r], sBv[st * kTileN + nl * kR + r]));
                const int64_t j = sJ[st * kNodes + nl];
                const bool mb = (member >> nl) & 1u;
                if (ok && j >= 0) ex[j] = mb ? best : -INFINITY;
                if (mb) {
                    fmax = fmaxf(fmax, best);
                    ++fcnt;
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(smem_u32(&bar_acc_empty[st]));
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTileN));
}

}  // namespace

size_t score_tc_smem(int d) {
    return (size_t)(d / 64) * 128 * 128 * (1 + 2 * kPlanes) + 2 * kTileN * 4 + 2 * kNodes * 8 + 2 * kProducers * 4 +
           1024;
}

cudaError_t launch_score_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st) {
    ProfScope ps_("k_score_tc", st);
    const int lane_tiles = (b.n_gl + kTileM - 1) / kTileM;
    int nb = 148 / max(1, lane_tiles * b.n_groups);
    nb = nb < 1 ? 1 : nb;
    dim3 grid(nb, lane_tiles, b.n_groups);
    const size_t smem = score_tc_smem(b.d);
    if (b.d == 128) {
        cudaFuncSetAttribute(k_score_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_score_tc<128><<<grid, kThreads, smem, st>>>(b, w, it, scale);
    } else {
        cudaFuncSetAttribute(k_score_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_score_tc<64><<<grid, kThreads, smem, st>>>(b, w, it, scale);
    }
    return cudaGetLastError();
}

}  // namespace zha
