// zha_score_tc.cu - plane-estimate scoring on the 5th-generation tensor cores (tcgen05).
//
// Same quantity as k_score (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的:
// 取这些平面的最大值; wqu.guru, section "Building the tree"): for every lane of a
// (sequence, KV head) group and every candidate node j,
//     e_j = max_r ( s q.m_r(j) + b_r(j) ).
// When a group holds many lanes (many query tokens x GQA heads) this is a dense
// contraction D[lane][(node, r)] = sum_k Q[lane][k] m_r(j)[k], run here as
// tcgen05.mma kind::tf32 with M = 128 lanes, N = 8 nodes x 16 planes, K = d, fp32
// accumulators in tensor memory.
//
// Precision: Q is bf16, hence exact in tf32.  The f32 summary m is split into
// hi = m with its 13 low mantissa bits cleared (exact tf32) and lo = m - hi (exact in
// f32); two MMA passes accumulate Q.hi + Q.lo, leaving a relative error of about 2^-22
// on m (the truncation of lo) - float32-grade scores.
//
// Shared-memory operands use the canonical K-major 128-byte-swizzle layout: per K block
// of 32 f32, rows are 128 bytes apart, the 16-byte chunk c of row r sits at chunk
// c ^ (r % 8), 8-row groups are 1024 bytes apart (the descriptor's stride byte offset).
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr int kTileM = 128;          // lanes per tile (MMA M)
constexpr int kTileN = 64;           // rows (node, plane) per tile (MMA N)
constexpr int kR = 16;               // planes per node on this path
constexpr int kNodes = kTileN / kR;  // nodes per tile
constexpr int kProducers = 256;      // warps 0-7: load, split, stage
constexpr int kEpilogue = 128;       // warps 8-11: TMEM -> scores; lane 0 of warp 8 issues the MMAs
constexpr int kThreads = kProducers + kEpilogue;
constexpr int kMmaWarp = kProducers / 32;   // also allocates tensor memory
constexpr int kRing = 3;             // node tiles whose loads each producer keeps in flight
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

// Instruction descriptor: kind::tf32, f32 accumulate, A and B K-major, M x N.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTileN >> 3) << 17) |
                            ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
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

// Byte offset of (row, 16-byte chunk c of K block kb) in a [KB][rows][128 B] tile.
__device__ __forceinline__ uint32_t swz(int kb, int rows, int row, int c) {
    return (uint32_t)(kb * (rows * 128) + row * 128 + ((c ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) k_score_tc(Batch b, Work w, int it, float scale) {
    constexpr int KB = D / 32;                        // 128-byte K blocks
    constexpr int A_BYTES = KB * kTileM * 128;
    constexpr int B_BYTES = KB * kTileN * 128;        // one plane of one stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = base;
    unsigned char* sB0 = base + A_BYTES;                                  // [2 stages][hi, lo][B_BYTES]
    float* sBv = reinterpret_cast<float*>(sB0 + 4 * B_BYTES);            // [2][kTileN] b values
    int64_t* sJ = reinterpret_cast<int64_t*>(sBv + 2 * kTileN);          // [2][kNodes] node ids (-1: none)
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
    // A: the tile's query rows as f32 (exact), zero rows past the group's lanes.
    for (int i = tid; i < kTileM * (D / 4); i += kThreads) {
        const int row = i / (D / 4), c4 = i % (D / 4);
        const int y = y0 + row;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (y < b.n_gl) {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(b.Q + lane_of(b, s, g, y) * D) + c4);
            const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
            const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
            v = make_float4(a0.x, a0.y, a1.x, a1.y);
        }
        *reinterpret_cast<float4*>(sA + swz(c4 / 8, kTileM, row, c4 % 8)) = v;
    }
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
        // ---------------- producers: rows of node tiles -> tf32 hi / f32 lo, swizzled.
        // Each thread keeps the loads of kRing tiles in flight (register ring, static slots).
        constexpr int kRowStep = kProducers / (D / 4);
        constexpr int kU = kTileN / kRowStep;
        const int c4 = tid % (D / 4);
        const int row0 = tid / (D / 4);
        auto prefetch = [&](int64_t i, float4 (&pre)[kU], float& preb, int64_t& prej) {
            if (i >= nt) return;
            const int64_t t = blockIdx.x + i * gridDim.x;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int row = row0 + u * kRowStep;
                const int64_t j = node_of(t, row / kR);
                pre[u] = j >= 0 ? __ldg(reinterpret_cast<const float4*>(recb + j * ns + (int64_t)(row % kR) * D) + c4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (tid < kTileN) {
                prej = node_of(t, tid / kR);
                preb = prej >= 0 ? __ldg(recb + prej * ns + (int64_t)kR * D + tid % kR) : 0.0f;
            }
        };
        // stage tile i from its ring slot, then refill the slot with tile i + kRing
        auto step = [&](int64_t i, float4 (&pre)[kU], float& preb, int64_t& prej) -> bool {
            if (i >= nt) return false;
            const int st = (int)(i & 1);
            // stage st (and its b / node ids) is free once the epilogue of tile i-2 is done
            if (i >= 2 && !mbar_wait(smem_u32(&bar_acc_empty[st]), (uint32_t)(((i >> 1) - 1) & 1))) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (abort_sh) return false;
            unsigned char* hiB = sB0 + (2 * st) * B_BYTES;
            unsigned char* loB = hiB + B_BYTES;
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int row = row0 + u * kRowStep;
                const float4 m = pre[u];
                float4 hi, lo;
                hi.x = __uint_as_float(__float_as_uint(m.x) & 0xFFFFE000u); lo.x = m.x - hi.x;
                hi.y = __uint_as_float(__float_as_uint(m.y) & 0xFFFFE000u); lo.y = m.y - hi.y;
                hi.z = __uint_as_float(__float_as_uint(m.z) & 0xFFFFE000u); lo.z = m.z - hi.z;
                hi.w = __uint_as_float(__float_as_uint(m.w) & 0xFFFFE000u); lo.w = m.w - hi.w;
                const uint32_t off = swz(c4 / 8, kTileN, row, c4 % 8);
                *reinterpret_cast<float4*>(hiB + off) = hi;
                *reinterpret_cast<float4*>(loB + off) = lo;
            }
            if (tid < kTileN) {
                sBv[st * kTileN + tid] = preb;
                if (tid % kR == 0) sJ[st * kNodes + tid / kR] = prej;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(smem_u32(&bar_full[st]));
            prefetch(i + kRing, pre, preb, prej);
            return true;
        };
        float4 p0[kU], p1[kU], p2[kU];
        float b0 = 0.f, b1 = 0.f, b2 = 0.f;
        int64_t j0 = -1, j1 = -1, j2 = -1;
        prefetch(0, p0, b0, j0);
        prefetch(1, p1, b1, j1);
        prefetch(2, p2, b2, j2);
        for (int64_t i = 0; i < nt; i += kRing) {
            if (!step(i, p0, b0, j0)) break;
            if (!step(i + 1, p1, b1, j1)) break;
            if (!step(i + 2, p2, b2, j2)) break;
        }
    } else {
        // ---------------- epilogue: scores of tile i from accumulator i % 2.  Lane 0 of the
        // first epilogue warp issues tile i+1's MMAs before this warp drains tile i.
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int y = y0 + row;
        const bool ok = y < b.n_gl;
        const int64_t x = lane_of(b, s, g, ok ? y : 0);
        float* ex = w.e + x * w.es;
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
            const uint32_t h0 = smem_u32(sB0 + (2 * st) * B_BYTES), l0 = h0 + B_BYTES;
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                const uint32_t b0 = pass == 0 ? h0 : l0;
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_tf32(d, umma_desc(a0 + kb * (kTileM * 128) + kk * 32),
                                 umma_desc(b0 + kb * (kTileN * 128) + kk * 32), (pass | kb | kk) ? 1u : 0u);
            }
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
            if (abort_sh) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) {
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(st * kTileN + nl * kR), v);
                float best = -INFINITY;
#pragma unroll
                for (int r = 0; r < kR; ++r) best = fmaxf(best, fmaf(scale, v[r], sBv[st * kTileN + nl * kR + r]));
                const int64_t j = sJ[st * kNodes + nl];
                if (ok && j >= 0) ex[j] = best;
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(smem_u32(&bar_acc_empty[st]));
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
    return (size_t)(d / 32) * 128 * (kTileM + 4 * kTileN) + 2 * kTileN * 4 + 2 * kNodes * 8 + 1024;
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
