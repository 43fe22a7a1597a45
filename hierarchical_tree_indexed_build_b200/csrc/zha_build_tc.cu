// zha_build_tc.cu - tree build on the 5th-generation tensor cores (tcgen05), fed by TMA.
//
// What is computed (pages: "Zyphra ZHA 稀疏注意力…" fluxbbs.com, section 树形索引是怎么搭的;
// "Zyphra发布层级注意力ZHA…" wqu.guru, section "Building the tree"): for chunk j of C tokens of
// KV head g and reference query q_r,
//     a_t = s q_r.k_t,   lse_r = log sum_t exp(a_t),   m_r = sum_t exp(a_t - lse_r) k_t,
//     b_r = lse_r - s q_r.m_r,
// and each level above merges its C children with the online-softmax combine.
//
// Geometry of this kernel: C = 4, R = 16, d = 64 or 128 (the deep trees), summaries as fp16
// hi + lo planes; other geometries and formats use the CUDA-core streaming build.  A CTA
// works on one KV head, persistent over tiles of 128 tokens.  A tile is 4 groups of 8 chunks (32 tokens).  For each group:
//   MMA 1    S[(r, j)][t] = q_r . k_t for the group's 32 tokens (M = 128 rows r*8 + j, every
//            row r*8 + j holding q_r; N = 32 tokens; K = d): bf16 x bf16 products, f32 sums.
//   softmax  the thread owning row (r, j) takes the 4 scores of chunk j: lse_r(j) and the
//            weights w_t = exp(a_t - lse_r(j)), each split into three bf16 terms w = hi + mid
//            + lo (24 significant bits, float32-grade), written into row r*8 + j of three
//            K-major weight planes in shared memory (the row's other columns stay 0).  Since s q_r.m_r = sum_t w_t a_t, the
//            same thread has b_r(j) = lse_r(j) - sum_t w_t a_t without a dot product.
//   MMA 2    m[(r, j)][k] = sum_t W[(r, j)][t] K[t][k] in three passes (hi, mid, lo), the tile's K
//            rows taken as an MN-major operand - the same shared-memory bytes MMA 1 reads
//            K-major.
//   records  the same thread encodes m_r(j) as the fp16 hi + lo planes of the node record and
//            folds level 2 (4 chunks = the rows of 4 neighbouring lanes: a butterfly
//            reduce-scatter, each lane keeping a quarter of the dimensions) and level 3 (16
//            chunks = two groups: the first group's level-2 rows pass through shared memory
//            to the warpgroup that takes the second).  The parents' b follow from the children's:
//            s q_r.m_r(P) = sum_c exp(lse_c - lse_P) (lse_c - b_c).  Levels above 3 come from
//            k_merge.
// A node's summary depends only on its own rows of K (other rows enter with weight exactly
// 0 and rows past the cache read as 0), so a tile recomputed by an append gives the same
// bits as the full build.
//
// Warp roles (448 threads): warp 0 TMA loads of K tiles; warp 1 MMA issue (one thread);
// epilogue warpgroups 0, 1, 2 (warps 2-5, 6-9, 10-13) take groups q = w, w + 3, ... of the
// CTA's sequence; each owns a pair of tensor-memory buffers (S: 32 columns, m: d columns) and
// three weight planes of 32 tokens (warpgroups 0 and 1 share one set of 128-byte rows, each
// its half).  Three warpgroups keep more record stores in flight than two.  The level-3
// exchange goes through one of two shared-memory buffers by the parity of the group pair.
// Every wait is bounded (about 2 s); a wait that gives up sets bit 1 of the tree's flag word
// (the routing calls report it as a device status) and the CTA drains and leaves.
#include <math.h>

#include <algorithm>

#include <cudaTypedefs.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr int kC = 4;                 // tokens per chunk
constexpr int kR = 16;                // reference queries
constexpr int kTileTok = 128;         // tokens per tile
constexpr int kGroupChunks = 128 / kR;               // 8 chunks per MMA row block
constexpr int kGroupTok = kGroupChunks * kC;         // 32 tokens
constexpr int kGroups = kTileTok / kGroupTok;        // 4 groups per tile
constexpr int kStagesK = 2;           // K tiles in flight
constexpr int kWPlanes = 3;           // bf16 terms of each weight
constexpr int kBlk = 128 * 128;       // bytes of a 128-row block of 128-byte rows
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int32_t kFlagRange = 1;     // tree flag bits
constexpr int32_t kFlagTimeout = 2;

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16, bf16 A and B, f32 D, M = 128, N = n, A K-major; b_mn: B is MN-major.
__host__ __device__ constexpr uint32_t idesc(int n, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d), "l"(a), "l"(b), "r"(id), "r"(acc));
}

__device__ __forceinline__ void commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Waits for the phase with the given parity; false after about 2 s.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
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

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        :
        : "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(mbar)
        : "memory");
}

// Starts the load of 32 consecutive columns of this thread's tensor-memory lane into r; the
// registers hold the values only after tld_wait(r).
__device__ __forceinline__ void tld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
// The wait for it, with the loaded registers as its operands, so that no use of them can be
// scheduled before it.
__device__ __forceinline__ void tld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                   "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

__device__ __forceinline__ void tld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    tld32_issue(taddr, r);
    tld_wait(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Byte offset of 16-byte chunk c16 of row r in a K-major tile of 128-byte rows (128B swizzle).
__device__ __forceinline__ uint32_t kmaj(int r, int c16) {
    return (uint32_t)((c16 >> 3) * kBlk + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}

// Two weights as three bf16 terms each (round to nearest even, then the remainders): the
// sum of the terms is the f32 weight within 2^-24 of it.
__device__ __forceinline__ void split3_bf16x2(float a, float b, uint32_t (&t)[3]) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        const float2 hf = __bfloat1622float2(h);
        t[i] = *reinterpret_cast<const uint32_t*>(&h);
        a -= hf.x;
        b -= hf.y;
    }
}

// log(exp a + exp b), the same bits for (a, b) and (b, a).  The fast intrinsics (relative
// error about 2^-21) are far inside the summaries' 1e-4 bar.
__device__ __forceinline__ float lse2f(float a, float b) {
    const float m = fmaxf(a, b);
    return m + __logf(__expf(a - m) + __expf(b - m));
}

// One 32-byte store (a whole sector) of 8 32-bit words.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

// fp16 hi and lo planes of 16 consecutive m values at hp / lp (32 bytes each, 32-byte aligned).
__device__ __forceinline__ void store_planes16(const float* v, __half* hp, __half* lp, bool& bad) {
    uint32_t h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __half2 hh = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
        const float2 hf = __half22float2(hh);
        const __half2 ll = __floats2half2_rn(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
        h[i] = *reinterpret_cast<const uint32_t*>(&hh);
        l[i] = *reinterpret_cast<const uint32_t*>(&ll);
        bad |= !(fabsf(v[2 * i]) < 65504.0f) || !(fabsf(v[2 * i + 1]) < 65504.0f);
    }
    st_global_v8(hp, h);
    st_global_v8(lp, l);
}

// fp16 hi and lo planes of n consecutive m values at hp / lp (n = 8: 16 bytes each;
// n = 4: 8 bytes each); `bad` for |m| >= 65504.
template <int n>
__device__ __forceinline__ void store_planes(const float* v, __half* hp, __half* lp, bool& bad) {
    uint32_t h[n / 2], l[n / 2];
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
        const __half2 hh = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
        const float2 hf = __half22float2(hh);
        const __half2 ll = __floats2half2_rn(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
        h[i] = *reinterpret_cast<const uint32_t*>(&hh);
        l[i] = *reinterpret_cast<const uint32_t*>(&ll);
        bad |= !(fabsf(v[2 * i]) < 65504.0f) || !(fabsf(v[2 * i + 1]) < 65504.0f);
    }
    if constexpr (n == 8) {
        *reinterpret_cast<uint4*>(hp) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lp) = make_uint4(l[0], l[1], l[2], l[3]);
    } else {
        *reinterpret_cast<uint2*>(hp) = make_uint2(h[0], h[1]);
        *reinterpret_cast<uint2*>(lp) = make_uint2(l[0], l[1]);
    }
}

template <int D>
struct Smem {
    static constexpr int KB = D / 64;                     // 128-byte blocks of a K row
    static constexpr int kTileBytes = KB * kBlk;          // one K tile (128 tokens)
    static constexpr int kQBytes = KB * kBlk;             // q_r over 128 rows
    static constexpr int kWBytes = kBlk;                  // one weight plane (128 rows x 64 tokens)
    static constexpr int kXFloats = kR * 2 * D;           // level-2 exchange [r][P][d]
    // two sets of weight planes (warpgroups 0 and 1 in the halves of set 0, warpgroup 2 in
    // set 0's layout of set 1) and two level-3 exchange buffers
    static constexpr size_t bytes = (size_t)kStagesK * kTileBytes + kQBytes + 2 * kWPlanes * (size_t)kWBytes +
                                    2 * ((size_t)kXFloats * 4 + (size_t)kR * 2 * 2 * 4) + 1024;
};

constexpr int kEpiWG = 3;             // epilogue warpgroups
constexpr int kBuildThreads = 64 + 128 * kEpiWG;

template <int D>
__global__ void __launch_bounds__(kBuildThreads, 1) k_build_tc(const __grid_constant__ CUtensorMap kmap, BuildTcArgs a) {
    using S = Smem<D>;
    constexpr int KB = S::KB;
    constexpr uint32_t kColS = 0;          // S of warpgroup w: columns 32 w
    constexpr uint32_t kColM = 32 * kEpiWG;   // m of warpgroup w: columns 96 + w D
    constexpr uint32_t kCols = 512;
    static_assert(kColM + 2 * D <= kCols, "tensor memory");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sK = base;                                       // [kStagesK][tile]
    unsigned char* sQ = sK + kStagesK * S::kTileBytes;              // A of MMA 1
    unsigned char* sW = sQ + S::kQBytes;                            // [set][plane][kWBytes]
    float* sX0 = reinterpret_cast<float*>(sW + 2 * kWPlanes * S::kWBytes);  // [2] level-2 exchange [r][P][D]
    float* sXl0 = sX0 + 2 * S::kXFloats;                            // [2] its (lse, s q.m) [r][P][2]
    __shared__ __align__(8) uint64_t bK_full[kStagesK], bK_empty[kStagesK], bS_full[kEpiWG], bS_empty[kEpiWG],
        bW_full[kEpiWG], bM_full[kEpiWG], bM_empty[kEpiWG], bX_full[2], bX_empty[2], bDone;
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_flag;
    volatile int& abort_sh = abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hg = blockIdx.y;                                       // KV head of this CTA
    const int64_t ntiles = a.t1 - a.t0;
    if ((int64_t)blockIdx.x >= ntiles) return;                       // whole CTA, before any barrier
    const int nt = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_sh)), "r"(kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < kStagesK; ++i) {
            mbar_init(su32(&bK_full[i]), 1);
            mbar_init(su32(&bK_empty[i]), 1);
        }
        for (int i = 0; i < kEpiWG; ++i) {
            mbar_init(su32(&bS_full[i]), 1);
            mbar_init(su32(&bS_empty[i]), 128);
            mbar_init(su32(&bW_full[i]), 128);
            mbar_init(su32(&bM_full[i]), 1);
            mbar_init(su32(&bM_empty[i]), 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(su32(&bX_full[i]), 128);
            mbar_init(su32(&bX_empty[i]), 128);
        }
        mbar_init(su32(&bDone), 1);
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    // weight planes start at zero (a row only ever receives its own chunk's 4 columns); the
    // MMA-1 operand holds q_r in every row r*8 + j (K-major, 128B swizzle)
    for (int i = tid; i < 2 * kWPlanes * S::kWBytes / 16; i += blockDim.x) reinterpret_cast<uint4*>(sW)[i] = make_uint4(0, 0, 0, 0);
    const __nv_bfloat16* qg = a.qref + (int64_t)hg * kR * D;
    for (int i = tid; i < 128 * (D / 8); i += blockDim.x) {
        const int row = i / (D / 8), c16 = i % (D / 8);
        *reinterpret_cast<uint4*>(sQ + kmaj(row, c16)) = __ldg(reinterpret_cast<const uint4*>(qg + (row >> 3) * D) + c16);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_sh;

    if (warp == 0) {
        // ---------------- TMA loads of K tiles (one thread)
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&kmap) : "memory");
            int issued = 0;
            for (int i = 0; i < nt && !abort_sh; ++i) {
                const int st = i % kStagesK;
                if (i >= kStagesK && !mbar_wait(su32(&bK_empty[st]), (uint32_t)(((i / kStagesK) - 1) & 1))) {
                    atomicOr(a.rflag, kFlagTimeout);
                    abort_sh = 1;
                    break;
                }
                const int64_t t = a.t0 + blockIdx.x + (int64_t)i * gridDim.x;
                const uint32_t fb = su32(&bK_full[st]);
                mbar_expect_tx(fb, (uint32_t)S::kTileBytes);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_3d(su32(sK + (size_t)st * S::kTileBytes + kb * kBlk), &kmap, kb * 64, (int)(t * kTileTok), hg, fb);
                issued = i + 1;
            }
            // copies still in flight land before the CTA leaves
            for (int i = std::max(0, issued - kStagesK); i < issued; ++i)
                mbar_wait(su32(&bK_full[i % kStagesK]), (uint32_t)((i / kStagesK) & 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issue (one thread).  Group q = 4 i + g of tile i uses the
        // buffers of warpgroup q % 3 for the (q / 3)-th time.
        if (lane == 0) {
            const int nq = nt * kGroups;
            auto mma1 = [&](int q) -> bool {
                const int i = q / kGroups, g = q % kGroups, w = q % kEpiWG, u = q / kEpiWG, st = i % kStagesK;
                if (g == 0 && !mbar_wait(su32(&bK_full[st]), (uint32_t)((i / kStagesK) & 1))) return false;
                if (u >= 1 && !mbar_wait(su32(&bS_empty[w]), (uint32_t)((u - 1) & 1))) return false;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t k0 = su32(sK + (size_t)st * S::kTileBytes) + g * kGroupTok * 128;
                const uint32_t q0 = su32(sQ);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t off = kb * kBlk + kk * 32;
                        mma(tmem + kColS + w * 32, desc_sw128(q0 + off, 16, 1024), desc_sw128(k0 + off, 16, 1024),
                            idesc(kGroupTok, 0), (kb | kk) ? 1u : 0u);
                    }
                commit(su32(&bS_full[w]));
                return true;
            };
            auto mma2 = [&](int q) -> bool {
                const int i = q / kGroups, g = q % kGroups, w = q % kEpiWG, u = q / kEpiWG, st = i % kStagesK;
                if (!mbar_wait(su32(&bW_full[w]), (uint32_t)(u & 1))) return false;
                if (u >= 1 && !mbar_wait(su32(&bM_empty[w]), (uint32_t)((u - 1) & 1))) return false;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t k0 = su32(sK + (size_t)st * S::kTileBytes) + g * kGroupTok * 128;
#pragma unroll
                for (int pl = 0; pl < kWPlanes; ++pl) {
                    // warpgroup w's 32 tokens: bytes 64 (w & 1) .. of the rows of set w >> 1
                    const uint32_t a0 = su32(sW + ((w >> 1) * kWPlanes + pl) * S::kWBytes) + (w & 1) * 64;
#pragma unroll
                    for (int ks = 0; ks < kGroupTok / 16; ++ks)
                        mma(tmem + kColM + w * D, desc_sw128(a0 + ks * 32, 16, 1024),
                            desc_sw128(k0 + ks * 16 * 128, kBlk, 1024), idesc(D, 1), (pl | ks) ? 1u : 0u);
                }
                commit(su32(&bM_full[w]));
                if (g == kGroups - 1) commit(su32(&bK_empty[st]));   // the tile's last reader
                return true;
            };
            bool ok = nq > 0 ? mma1(0) : true;
            for (int q = 0; q < nq && ok && !abort_sh; ++q) {
                if (q + 1 < nq) ok = mma1(q + 1);
                if (ok) ok = mma2(q);
            }
            if (!ok) {
                atomicOr(a.rflag, kFlagTimeout);
                abort_sh = 1;
            }
            // every MMA issued above has completed before tensor memory is released
            commit(su32(&bDone));
            mbar_wait(su32(&bDone), 0);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue warpgroups: thread = TMEM lane r*8 + j
        const int w = (warp - 2) >> 2;                       // warpgroup: groups q with q % 3 == w
        const int quad = warp & 3;                           // TMEM lane quarter of this warp
        const int row = quad * 32 + lane;
        const int r = row >> 3, j = row & 7;
        const int P = j >> 2, c4 = j & 3;                   // level-2 node of the group, lane within it
        const uint32_t tl = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + tl + kColS + w * 32;
        const uint32_t tM = tmem + tl + kColM + w * D;
        unsigned char* wPl = sW + (w >> 1) * kWPlanes * S::kWBytes;   // this warpgroup's weight planes
        // tokens 4j .. 4j+3 of the row, in this warpgroup's 64-byte half of the 128-byte row
        const uint32_t woff = kmaj(row, (j >> 1) + 4 * (w & 1)) + (j & 1) * 8;
        const int nq = nt * kGroups;
        bool bad = false;
        auto give_up = [&]() {
            atomicOr(a.rflag, kFlagTimeout);
            abort_sh = 1;
        };
        for (int q = w; q < nq; q += kEpiWG) {
            const int i = q / kGroups, g = q % kGroups, u = q / kEpiWG;
            // level-3 exchange of group pair q >> 1: buffer (q >> 1) & 1, its (q >> 2)-th use
            const int xb = (q >> 1) & 1;
            const uint32_t xuse = (uint32_t)(q >> 2);
            float* sX = sX0 + xb * S::kXFloats;
            float* sXl = sXl0 + xb * (kR * 2 * 2);
            const int64_t t = a.t0 + blockIdx.x + (int64_t)i * gridDim.x;
            // -- scores of chunk j, softmax, weights, b
            if (!mbar_wait(su32(&bS_full[w]), (uint32_t)(u & 1))) give_up();
            if (__any_sync(0xffffffffu, abort_sh != 0)) break;   // warp-uniform: tcgen05.ld is collective
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            float sv[32];
            tld32(tS, sv);
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(su32(&bS_empty[w]));
            float av[kC];
#pragma unroll
            for (int c = 0; c < kC; ++c) av[c] = sv[c];
#pragma unroll
            for (int jj = 1; jj < kGroupChunks; ++jj)
                if (jj == j)
#pragma unroll
                    for (int c = 0; c < kC; ++c) av[c] = sv[jj * kC + c];
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                av[c] *= a.scale;
                mx = fmaxf(mx, av[c]);
            }
            float z = 0.0f, ev[kC];
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                ev[c] = __expf(av[c] - mx);
                z += ev[c];
            }
            const float l1 = mx + __logf(z);
            const float iz = 1.0f / z;
            float wv[kC], wa = 0.0f;                        // wa = s q_r.m_r = sum_t w_t a_t
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                wv[c] = ev[c] * iz;
                wa = fmaf(wv[c], av[c], wa);
            }
            uint32_t t01[3], t23[3];
            split3_bf16x2(wv[0], wv[1], t01);
            split3_bf16x2(wv[2], wv[3], t23);
#pragma unroll
            for (int pl = 0; pl < kWPlanes; ++pl)
                *reinterpret_cast<uint2*>(wPl + pl * S::kWBytes + woff) = make_uint2(t01[pl], t23[pl]);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(su32(&bW_full[w]));

            // -- the log-masses and weights of the levels above (lanes 4P .. 4P+3 are the 4
            // chunks of level-2 node P; the group pair (g even, g odd) forms a level-3 node)
            const int64_t j1 = t * (kTileTok / kC) + g * kGroupChunks + j;
            const int64_t j2 = t * (kTileTok / (kC * kC)) + g * 2 + P;
            const int64_t j3 = t * 2 + (g >> 1);
            const bool st1 = j1 < a.n1, st2 = a.k_emit >= 2 && j2 < a.n2, st3 = a.k_emit >= 3 && j3 < a.n3;
            float l2 = lse2f(l1, __shfl_xor_sync(0xffffffffu, l1, 1));
            l2 = lse2f(l2, __shfl_xor_sync(0xffffffffu, l2, 2));
            const float w21 = __expf(l1 - l2);
            float wa2 = w21 * wa;                            // s q_r.m_r of the level-2 node
            wa2 += __shfl_xor_sync(0xffffffffu, wa2, 1);
            wa2 += __shfl_xor_sync(0xffffffffu, wa2, 2);
            const bool second = (g & 1) != 0;
            const bool lv3 = a.k_emit >= 3;
            float l3 = 0.0f, wX0 = 0.0f, wX1 = 0.0f, w32 = 0.0f, wa3 = 0.0f;
            if (lv3 && second) {
                if (!mbar_wait(su32(&bX_full[xb]), xuse & 1u)) give_up();
                const float la0 = sXl[(r * 2 + 0) * 2], la1 = sXl[(r * 2 + 1) * 2];
                const float lo = __shfl_xor_sync(0xffffffffu, l2, 4);   // this group's other level-2 node
                l3 = lse2f(lse2f(la0, la1), lse2f(l2, lo));
                wX0 = __expf(la0 - l3);
                wX1 = __expf(la1 - l3);
                w32 = __expf(l2 - l3);
                float y = w32 * wa2;
                y += __shfl_xor_sync(0xffffffffu, y, 4);
                wa3 = fmaf(wX0, sXl[(r * 2 + 0) * 2 + 1], wX1 * sXl[(r * 2 + 1) * 2 + 1]) + y;
            }
            if (lv3 && !second && xuse >= 1) {
                // the second group of this buffer's previous pair has read it
                if (!mbar_wait(su32(&bX_empty[xb]), (xuse - 1) & 1u)) give_up();
            }

            if (!mbar_wait(su32(&bM_full[w]), (uint32_t)(u & 1))) give_up();
            if (__any_sync(0xffffffffu, abort_sh != 0)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            __half* r1 = reinterpret_cast<__half*>(a.rec[1] + ((int64_t)hg * a.cap[1] + j1) * a.ns);
            __half* r2 = a.k_emit >= 2 ? reinterpret_cast<__half*>(a.rec[2] + ((int64_t)hg * a.cap[2] + j2) * a.ns) : nullptr;
            __half* r3 = lv3 ? reinterpret_cast<__half*>(a.rec[3] + ((int64_t)hg * a.cap[3] + j3) * a.ns) : nullptr;
            const bool lo2 = (c4 & 2) == 0, lo1 = (c4 & 1) == 0;
            // pieces of 32 columns: the load of piece p + 1 is in flight while piece p is used
            uint32_t nx[32];
            tld32_issue(tM, nx);
            tld_wait(nx);
#pragma unroll 1
            for (int p = 0; p < D / 32; ++p) {
                float v[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(nx[k]);
                if (p + 1 < D / 32) tld32_issue(tM + (p + 1) * 32, nx);
                if (st1) {
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        store_planes16(v + 16 * e, r1 + r * D + p * 32 + 16 * e, r1 + kR * D + r * D + p * 32 + 16 * e, bad);
                }
                // level 2: sum over the 4 chunks of w21 * m, reduce-scattered so that lane c4
                // keeps dims 8 c4 .. 8 c4 + 7 of this piece
                float y[16], m2[8];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float keep = w21 * (lo2 ? v[k] : v[16 + k]);
                    const float give = w21 * (lo2 ? v[16 + k] : v[k]);
                    y[k] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float keep = lo1 ? y[k] : y[8 + k];
                    const float give = lo1 ? y[8 + k] : y[k];
                    m2[k] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
                }
                const int dim = p * 32 + 8 * c4;            // first of this lane's 8 dims
                if (st2) store_planes<8>(m2, r2 + r * D + dim, r2 + kR * D + r * D + dim, bad);
                if (lv3) {
                    float* xrow = sX + (r * 2 + P) * D + dim;
                    if (!second) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) xrow[k] = m2[k];   // left for the partner warpgroup
                    } else {
                        const float* x0 = sX + (r * 2 + 0) * D + dim;
                        const float* x1 = sX + (r * 2 + 1) * D + dim;
                        float m3[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            float yy = w32 * m2[k];
                            yy += __shfl_xor_sync(0xffffffffu, yy, 4);
                            m3[k] = fmaf(wX0, x0[k], wX1 * x1[k]) + yy;
                        }
                        // lanes of node 0 store dims +0..3, lanes of node 1 dims +4..7 (static
                        // offsets: the array stays in registers)
                        if (st3) {
                            if (P == 0) store_planes<4>(m3, r3 + r * D + dim, r3 + kR * D + r * D + dim, bad);
                            else store_planes<4>(m3 + 4, r3 + r * D + dim + 4, r3 + kR * D + r * D + dim + 4, bad);
                        }
                    }
                }
                tld_wait(nx);                                // piece p + 1 has landed
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(su32(&bM_empty[w]));
            // b = lse - s q_r.m_r, and lse, of every stored node
            if (st1) {
                reinterpret_cast<float*>(r1)[kR * D + r] = l1 - wa;
                a.lse[1][((int64_t)hg * a.cap[1] + j1) * kR + r] = l1;
            }
            if (st2 && c4 == 0) {
                reinterpret_cast<float*>(r2)[kR * D + r] = l2 - wa2;
                a.lse[2][((int64_t)hg * a.cap[2] + j2) * kR + r] = l2;
            }
            if (lv3) {
                if (!second) {
                    if (c4 == 0) {
                        sXl[(r * 2 + P) * 2] = l2;
                        sXl[(r * 2 + P) * 2 + 1] = wa2;
                    }
                    mbar_arrive(su32(&bX_full[xb]));        // this pair's exchange is written
                } else {
                    if (st3 && j == 0) {
                        reinterpret_cast<float*>(r3)[kR * D + r] = l3 - wa3;
                        a.lse[3][((int64_t)hg * a.cap[3] + j3) * kR + r] = l3;
                    }
                    mbar_arrive(su32(&bX_empty[xb]));       // exchange read
                }
            }
        }
        if (bad) atomicOr(a.rflag, kFlagRange);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols));
}

// K viewed as (dim, token, KV head) with tokens [0, n_tokens): rows past the cache read as 0.
bool encode_k_map(CUtensorMap* map, const __nv_bfloat16* K, int d, int64_t ld, int64_t n_tokens, int Hkv) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n_tokens, (cuuint64_t)Hkv};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)ld * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTileTok, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(K), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool build_tc_supported(int C, int R, int d, int fmt) {
    return C == kC && R == kR && (d == 64 || d == 128) && fmt == kFmtF16x2;
}

cudaError_t launch_build_tc(const BuildTcArgs& a, int d, cudaStream_t st) {
    if (a.t1 <= a.t0 || a.n_tokens <= 0) return cudaSuccess;
    CUtensorMap map;
    if (!encode_k_map(&map, a.K, d, a.ld, a.n_tokens, a.Hkv)) return cudaErrorInvalidValue;
    const int64_t tiles = a.t1 - a.t0;
    const int per_head = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, std::max(1, sm_count() / a.Hkv)));
    const dim3 grid((unsigned)per_head, (unsigned)a.Hkv);
    ProfScope ps_("k_build_tc", st);
    if (d == 128) {
        const size_t smem = Smem<128>::bytes;
        cudaFuncSetAttribute(k_build_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_build_tc<128><<<grid, kBuildThreads, smem, st>>>(map, a);
    } else {
        const size_t smem = Smem<64>::bytes;
        cudaFuncSetAttribute(k_build_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_build_tc<64><<<grid, kBuildThreads, smem, st>>>(map, a);
    }
    return cudaGetLastError();
}

}  // namespace zha
