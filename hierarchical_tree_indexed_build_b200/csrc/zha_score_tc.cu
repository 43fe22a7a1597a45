// zha_score_tc.cu - plane-estimate scoring on the 5th-generation tensor cores (tcgen05).
//
// Same quantity as k_score (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的:
// the estimate is the largest of the planes; wqu.guru, section "Building the tree"): for every lane of a
// (sequence, KV head) group and every candidate node j on the lane's frontier,
//     e_j = max_r ( s q.m_r(j) + b_r(j) ),
// and -inf for candidates off the lane's frontier (children of nodes other lanes kept).
// When a group holds many lanes (query tokens x GQA heads) this is a dense contraction
// D[lane][(node, r)] = sum_k Q[lane][k] m_r(j)[k], run here as tcgen05.mma kind::f16 with
// M = 128 lanes, N = 8 nodes x 16 planes, K = d, f32 accumulators in tensor memory.
//
// Precision: Q is bf16, which fp16 holds exactly for magnitudes in [2^-17, 65504).  The
// tree stores each summary m as two fp16 planes m = hi + lo (lo the fp16 rounding of
// m - hi), so two MMA passes accumulate Q.m exactly as the f32 scorer would see the stored
// m: float32-grade scores.  A query entry of magnitude >= 65504 does not fit; the kernel
// then sets kStatusRange (as does a tree whose summaries left the fp16 range).
//
// Pipeline (one CTA per SM, persistent over its node tiles of 8 nodes; LT = 1 or 2 lane
// tiles of 128 lanes per CTA share every node tile):
//   warp 0      loader: TMA copies of the nodes' two fp16 planes (boxes of 64 dims x 16
//               planes x 4 consecutive nodes, 128-byte swizzled by the copy engine into the
//               MMA operand layout; 1-node boxes when C is not a multiple of 4), of their b
//               values, and of the CTA lanes' membership words, into one of 3 stages;
//   warp 1      MMA issuer: per lane tile, 2 planes x d/16 tcgen05.mma kind::f16 with the
//               query tile (A) in tensor memory and the node tile (B) in shared memory;
//   warps 2..   epilogue, 4 per lane tile: tensor memory -> max over planes + b -> scores.
// With A in tensor memory an MMA reads only its B rows from shared memory.  Each lane tile
// job (node tile, lane tile) takes the next of three accumulators in turn, so the MMAs of
// up to two further jobs run while one job's epilogue drains.
// Tensor memory: accumulators at columns 0, 128 and 256, the queries of lane tile t at
// columns 384 + t d/2 (two fp16 of a row per 32-bit column).
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

size_t score_tc_smem_lt(int d, int lt, int planes);

namespace {

constexpr int kTileM = 128;          // lanes per tile (MMA M)
constexpr int kTileN = 128;          // rows (node, plane) per tile (MMA N)
constexpr int kR = 16;               // planes per node on this path
constexpr int kNodes = kTileN / kR;  // nodes per tile
// planes of m per record: two fp16 terms (hi, lo) or one bf16 plane
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

// Instruction descriptor: kind::f16 with fp16 (or, with bf, bf16) A/B, f32 accumulate, both
// K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_score(bool bf) {
    return (1u << 4) | (bf ? (1u << 7) | (1u << 10) : 0u) | ((uint32_t)(kTileN >> 3) << 17) |
           ((uint32_t)(kTileM >> 4) << 24);
}

// D (tensor memory) = or += A (tensor memory) x B (shared memory descriptor)
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "r"(tmem_a), "l"(b), "r"(id), "r"(acc));
}

// Writes 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :
        : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
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

// 32 x 32 bit transpose across a warp: lane y holds row y (bit t = element (y, t)); the result
// in lane t is column t (bit y = element (y, t)).  Five butterfly stages exchange ever smaller
// blocks with the partner lane (16, 8, 4, 2, 1 apart): about a quarter of the instructions of
// 32 ballots.
__device__ __forceinline__ uint32_t transpose32(uint32_t v, int lane) {
    const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int j = 16 >> k;
        const uint32_t m = masks[k];
        const uint32_t t = __shfl_xor_sync(0xffffffffu, v, j);
        v = (lane & j) ? ((v & ~m) | ((t & ~m) >> j)) : ((v & m) | ((t & m) << j));
    }
    return v;
}

// Lanes' kept bits of one level, transposed over the group's union list of that level:
// memb[grp][u][w] bit t = lane 32 w + t kept union node u.  Mode 0: the level above the one
// routing iteration `it` scores (its nodes are the candidates' parents); mode 1: level 1
// (the chunks attention gathers).  A block transposes a tile of 256 union entries x 256
// lanes (8 lane words): where the tile's entries are 256 consecutive nodes (a dense stretch
// of the union), each lane reads the 9 bitmap words covering them and realigns them by
// funnel shifts, warps transpose 32 x 32 bit blocks (butterfly shuffles) through shared memory, and
// each entry's 8 words are written as one 32-byte segment.  A tile whose entries lie within
// 1,024 nodes stages each lane's words of that window and transposes entry by entry from
// shared memory; sparser tiles read each entry's word from global memory.
// Grid (tiles, lane-word groups of 8, groups), 256 threads.
__global__ void __launch_bounds__(256) k_member(Batch b, Work w, int it, int mode) {
    __shared__ uint32_t T[256][33];                   // [lane][bitmap word of the tile's node window], padded
    __shared__ __align__(16) uint32_t O[256][8];      // [entry][lane word]
    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    int pl;
    if (mode == 0) {
        const int lev = sq.L - it;
        if (lev < 1 || lev == sq.L) return;           // top level: no parents
        pl = lev + 1;
    } else {
        if (sq.T == 0) return;                        // dense attention: no union
        pl = 1;
    }
    const int nu = w.ucount[grp];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lw0 = blockIdx.y * 8;
    const int y = lw0 * 32 + tid;                     // this thread's lane (load phase)
    const bool yok = y < b.n_gl;
    const uint32_t* kb = w.kept[pl] + lane_of(b, s, g, yok ? y : 0) * w.W[pl];
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    uint32_t* out = w.memb + (int64_t)grp * w.ms * w.mwords + lw0;
    for (int tx = blockIdx.x; tx * 256 < nu; tx += gridDim.x) {
        const int u0 = tx * 256, cnt = min(256, nu - u0);
        const int p0 = __ldg(ul + u0), pn = __ldg(ul + u0 + cnt - 1);
        const bool dense = cnt == 256 && pn == p0 + 255;   // 256 consecutive nodes; uniform in the block
        if (dense) {
            // the lane's 256 bits for nodes p0 .. p0 + 255: 9 words realigned by funnel shifts
            const int w0 = p0 >> 5, sh = p0 & 31;
            const int64_t W = w.W[pl];
            uint32_t wv[9];
#pragma unroll
            for (int k = 0; k < 9; ++k) wv[k] = (yok && w0 + k < W) ? __ldg(kb + w0 + k) : 0u;
#pragma unroll
            for (int k = 0; k < 8; ++k) T[tid][k] = __funnelshift_r(wv[k], wv[k + 1], sh);
            __syncthreads();
            // warp i: node word i of the tile, for each of the 8 lane words
#pragma unroll 2
            for (int lw = 0; lw < 8; ++lw) O[warp * 32 + lane][lw] = transpose32(T[lw * 32 + lane][warp], lane);
            __syncthreads();
            uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(u0 + tid) * w.mwords);
            dst[0] = make_uint4(O[tid][0], O[tid][1], O[tid][2], O[tid][3]);
            dst[1] = make_uint4(O[tid][4], O[tid][5], O[tid][6], O[tid][7]);
            __syncthreads();                          // T and O are reused by the next tile
        } else if (pn - p0 < 1024) {
            // the tile's entries lie in a window of <= 1,024 nodes: each lane stages the <= 33
            // bitmap words of the window once, then warps transpose entry by entry from there
            const int w0 = p0 >> 5, nw = (pn >> 5) - w0 + 1;
            const int64_t W = w.W[pl];
            for (int k = 0; k < nw; ++k) T[tid][k] = (yok && w0 + k < W) ? __ldg(kb + w0 + k) : 0u;
            __syncthreads();
            const int e0 = u0 + warp * 32;
            const int n = max(0, min(32, nu - e0));
            const int pmy = lane < n ? __ldg(ul + e0 + lane) : p0;
#pragma unroll 1
            for (int lw = 0; lw < 8; ++lw) {
                uint32_t mine = 0;
#pragma unroll 4
                for (int t = 0; t < 32; ++t) {
                    const int pt = __shfl_sync(0xffffffffu, pmy, t);
                    const uint32_t v = T[lw * 32 + lane][(pt >> 5) - w0];
                    const uint32_t r = __ballot_sync(0xffffffffu, (v >> (pt & 31)) & 1u);
                    if (lane == t) mine = r;
                }
                O[warp * 32 + lane][lw] = mine;
            }
            __syncthreads();
            if (tid < cnt) {
                uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(u0 + tid) * w.mwords);
                dst[0] = make_uint4(O[tid][0], O[tid][1], O[tid][2], O[tid][3]);
                dst[1] = make_uint4(O[tid][4], O[tid][5], O[tid][6], O[tid][7]);
            }
            __syncthreads();                          // T and O are reused by the next tile
        } else {
            // warp i: entries u0 + 32 i .., lane words lw0 .. lw0 + 7
            const int e0 = u0 + warp * 32;
            const int n = min(32, nu - e0);
            if (n > 0) {
                const int pmy = lane < n ? __ldg(ul + e0 + lane) : 0;
#pragma unroll 1
                for (int lw = 0; lw < 8; ++lw) {
                    const int yl = (lw0 + lw) * 32 + lane;
                    if ((lw0 + lw) * 32 >= b.n_gl) break;             // uniform in the warp
                    const bool ok = yl < b.n_gl;
                    const uint32_t* kl = w.kept[pl] + lane_of(b, s, g, ok ? yl : 0) * w.W[pl];
                    // all 32 entries' bits of this lane first (independent loads), then the transpose
                    uint32_t bits = 0;
#pragma unroll
                    for (int t = 0; t < 32; ++t) {
                        const int pt = __shfl_sync(0xffffffffu, pmy, t);
                        if (t < n && ok) bits |= ((__ldg(kl + (pt >> 5)) >> (pt & 31)) & 1u) << t;
                    }
                    const uint32_t mine = transpose32(bits, lane);
                    if (lane < n) out[(int64_t)(e0 + lane) * w.mwords + lw] = mine;
                }
            }
        }
    }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
        :
        : "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(dst), "l"(map), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :
                 : "r"(dst), "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

constexpr int kStages = 3;           // shared-memory stages of node tiles

template <int D, int LT, bool BF>
__global__ void __launch_bounds__(64 + 128 * LT, 1) k_score_tc(Batch b, Work w, int it, float scale) {
    constexpr int kPlanes = BF ? 1 : 2;
    constexpr int kEpilogue = 128 * LT;
    constexpr int kLW = 4 * LT;                       // 32-lane membership words per CTA
    constexpr int KB = D / 64;                        // 128-byte K blocks of 16-bit values
    constexpr int P_BYTES = KB * kTileN * 128;        // one plane of one stage
    constexpr int STAGE = kPlanes * P_BYTES;
    constexpr uint32_t kId = idesc_score(BF);
    constexpr int kBOff = BF ? kR * D / 2 : kR * D;   // floats from a record to its b values
    constexpr int kAcc = 3;                           // accumulator slots (columns 0, 128, 256)
    constexpr uint32_t kColA = kAcc * kTileN;         // queries after the accumulators
    constexpr uint32_t kCols = 512;
    static_assert(kColA + LT * (D / 2) <= kCols, "accumulators and queries must fit the 512 TMEM columns");
    constexpr uint32_t kNodeBytes = kPlanes * KB * 16 * 128;   // both planes of one node
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned start, reached by pointer arithmetic on the shared array so that every
    // pointer derived from it stays a shared-memory pointer (plain shared loads and stores)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sB0 = base;                                             // [kStages][2 planes][P_BYTES]
    float* sBv = reinterpret_cast<float*>(sB0 + kStages * STAGE);          // [kStages][kNodes][16] b values
    uint32_t* sMask = reinterpret_cast<uint32_t*>(sBv + kStages * kTileN); // [kStages][kNodes][kLW] membership
    int32_t* sJ = reinterpret_cast<int32_t*>(sMask + kStages * kNodes * kLW);   // [kStages][kNodes] node ids
    __shared__ __align__(8) uint64_t bar_full[kStages], bar_empty[kStages], bar_acc_full[kAcc], bar_acc_empty[kAcc];
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
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        atomicAdd(&w.ctr[kCtrUnionNodes + lev], (unsigned long long)nc);
        tree_flag_status(*sq.rflag, w.status);
    }
    const int ntiles = (nc + kNodes - 1) / kNodes;
    if ((int)blockIdx.x >= ntiles) return;          // whole block leaves before any barrier
    const int nt = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;   // tiles of this block
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y0 = blockIdx.y * (kTileM * LT);
    const bool runs = top || (C % 4 == 0);

    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&bar_full[i]), 1);
            mbar_init(smem_u32(&bar_empty[i]), kEpilogue);
        }
        for (int i = 0; i < kAcc; ++i) {
            mbar_init(smem_u32(&bar_acc_full[i]), 1);
            mbar_init(smem_u32(&bar_acc_empty[i]), kTileM);   // one lane tile drains a slot
        }
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_sh;

    // epilogue thread <-> one lane row of the CTA (TMEM lane quarter = warp % 4)
    const int ew = warp - 2;
    const int lt = ew >> 2, quad = warp & 3;
    const int row = lt * kTileM + quad * 32 + lane;
    const uint32_t tlane = (uint32_t)(quad * 32) << 16;
    if (warp >= 2) {
        // A: this lane's query row into tensor memory - as fp16 (exact in range) against
        // fp16 planes, as its own bf16 bits against a bf16 plane; zero rows past the group's lanes
        const int y = y0 + row;
        const uint4* qp = reinterpret_cast<const uint4*>(b.Q + lane_of(b, s, g, y < b.n_gl ? y : 0) * D);
        float amax = 0.0f;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            uint32_t hv[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (y < b.n_gl) v = __ldg(qp + h * 8 + c);
                const uint32_t* bv = &v.x;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if constexpr (BF) {
                        hv[c * 4 + t] = bv[t];
                    } else {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(bv + t));
                        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
                        const __half2 hh = __floats2half2_rn(f.x, f.y);
                        hv[c * 4 + t] = *reinterpret_cast<const uint32_t*>(&hh);
                    }
                }
            }
            tmem_st32(tmem + tlane + kColA + (uint32_t)(lt * (D / 2) + h * 32), hv);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        if (!(amax < kHalfMax)) atomicOr(w.status, kStatusRange);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    if (warp == 0) {
        // ---------------- loader.  Lanes compute the node ids of 4 tiles at a time (one
        // candidate each), a batch ahead of use; lane 0 issues the copies.
        const CUtensorMap* maps = w.tmaps + ((int64_t)s * (kMaxL + 1) + lev) * kMapsPerLevel;
#pragma unroll
        for (int k = 0; k < kMapsPerLevel; ++k)
            asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(maps + k) : "memory");
        // candidates come in aligned runs of 4 consecutive nodes with one parent when C % 4 == 0
        // (and at the top level): one 4-node box per plane and K block, one for b, one
        // membership row per run
        const float* recb = sq.rec[lev];
        const int64_t node0 = (int64_t)g * sq.cap[lev];               // first node of this KV head
        const int32_t* ul = w.ulist + (int64_t)grp * w.us;
        const uint32_t* memb = w.memb + (int64_t)grp * w.ms * w.mwords + (int64_t)blockIdx.y * kLW;
        auto ids = [&](int i0, int& j, int& u) {
            const int t = i0 + lane / kNodes;
            j = -1;
            u = 0;
            if (t < nt) {
                const int k = (blockIdx.x + t * gridDim.x) * kNodes + lane % kNodes;
                if (k < nc) {
                    if (top) {
                        j = k;
                    } else {
                        u = (int)((uint32_t)k / (uint32_t)C);
                        j = __ldg(ul + u) * C + (k - u * C);
                    }
                }
            }
        };
        int jc, uc, jn, un;
        ids(0, jc, uc);
        int issued = 0;
        bool stop = false;
        for (int i0 = 0; i0 < nt && !stop; i0 += 4) {
            ids(i0 + 4, jn, un);                      // next batch, in flight while this one issues
            for (int t = 0; t < 4 && i0 + t < nt; ++t) {
                const int i = i0 + t, st = i % kStages;
                const int src = lane < kNodes ? t * kNodes + lane : 0;
                const int jj = __shfl_sync(0xffffffffu, jc, src);   // lanes 0..7: node nl = lane
                const int uu = __shfl_sync(0xffffffffu, uc, src);
                if (lane == 0 && i >= kStages && !abort_sh &&
                    !mbar_wait(smem_u32(&bar_empty[st]), (uint32_t)(((i / kStages) - 1) & 1))) {
                    atomicOr(w.status, kStatusTimeout);
                    abort_sh = 1;
                }
                if (__any_sync(0xffffffffu, abort_sh != 0)) {
                    stop = true;
                    break;
                }
                uint32_t valid = __ballot_sync(0xffffffffu, lane < kNodes && jj >= 0);
                if (runs) valid &= 0x11u;                  // a run is loaded whole from its first node
                if (lane < kNodes) sJ[st * kNodes + lane] = jj;
                const uint32_t fb = smem_u32(&bar_full[st]);
                __syncwarp();
                if (lane == 0) {
                    // the stage's only arrival, with the bytes every copy below will deliver
                    const uint32_t per = runs ? 4 * kNodeBytes + 4 * kR * 4 : kNodeBytes + kR * 4;
                    mbar_expect_tx(fb, (uint32_t)__popc(valid) * (per + (top ? 0 : kLW * 4)));
                    const uint32_t sb = smem_u32(sB0 + (size_t)st * STAGE);
                    for (int nl = 0; nl < kNodes; ++nl) {
                        if (!((valid >> nl) & 1u)) continue;
                        const int wn = (int)(node0 + sJ[st * kNodes + nl]);
#pragma unroll
                        for (int pl = 0; pl < kPlanes; ++pl)
#pragma unroll
                            for (int kb = 0; kb < KB; ++kb)
                                tma_load_4d(sb + pl * P_BYTES + kb * (kTileN * 128) + nl * (kR * 128), maps + (runs ? 1 : 0),
                                            kb * 64, 0, pl, wn, fb);
                        if (runs)
                            tma_load_2d(smem_u32(sBv + st * kTileN + nl * kR), maps + 2, 0, wn, fb);
                        else
                            bulk_load(smem_u32(sBv + st * kTileN + nl * kR), recb + (int64_t)wn * sq.ns + kBOff, kR * 4, fb);
                    }
                }
                __syncwarp();
                // membership words of node (or run) nl = lane: row of its union parent uu
                if (!top && lane < kNodes && ((valid >> lane) & 1u))
                    bulk_load(smem_u32(sMask + (st * kNodes + lane) * kLW), memb + (int64_t)uu * w.mwords, kLW * 4, fb);
                __syncwarp();
                issued = i + 1;
            }
            jc = jn;
            uc = un;
        }
        // copies still in flight must land before the block ends
        if (lane == 0)
            for (int i = max(0, issued - kStages); i < issued; ++i)
                mbar_wait(smem_u32(&bar_full[i % kStages]), (uint32_t)((i / kStages) & 1));
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: the whole warp waits, one elected lane issues (a
        // converged warp issues tcgen05.mma at about twice the rate of a lone thread)
        {
            const int jobs = nt * LT;
            for (int q = 0; q < jobs; ++q) {
                if (__any_sync(0xffffffffu, abort_sh != 0)) break;
                const int i = q / LT, t = q % LT, st = i % kStages, slot = q % kAcc;
                bool okw = true;
                if (t == 0) okw = mbar_wait(smem_u32(&bar_full[st]), (uint32_t)((i / kStages) & 1));
                if (okw && q >= kAcc) okw = mbar_wait(smem_u32(&bar_acc_empty[slot]), (uint32_t)(((q / kAcc) - 1) & 1));
                if (!__all_sync(0xffffffffu, okw)) {
                    if (lane == 0) {
                        atomicOr(w.status, kStatusTimeout);
                        abort_sh = 1;
                    }
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                uint32_t leader;
                asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}\n" : "=r"(leader));
                if (leader) {
                    const uint32_t d = tmem + (uint32_t)(slot * kTileN);
                    const uint32_t ta = tmem + kColA + (uint32_t)(t * (D / 2));
                    const uint64_t db = umma_desc(smem_u32(sB0 + (size_t)st * STAGE));
#pragma unroll 1
                    for (int pk = 0; pk < kPlanes * KB; ++pk) {
                        const int pass = pk / KB, kb = pk % KB;
                        const uint64_t b1 = db + (uint64_t)((pass * P_BYTES + kb * (kTileN * 128)) >> 4);
                        const uint32_t a1 = ta + (uint32_t)(kb * 32);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16_ts(d, a1 + (uint32_t)(kk * 8), b1 + (uint64_t)(kk * 2), kId, (pk | kk) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bar_acc_full[slot]));
                }
                __syncwarp();
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue
        const int y = y0 + row;
        const bool ok = y < b.n_gl;
        const int64_t x = lane_of(b, s, g, ok ? y : 0);
        float* ex = w.e + x * w.es;
        float fmax = -INFINITY;
        int fcnt = 0;
#pragma unroll 1
        for (int i = 0; i < nt; ++i) {
            const int st = i % kStages, q = i * LT + lt, slot = q % kAcc;
            if (!mbar_wait(smem_u32(&bar_acc_full[slot]), (uint32_t)((q / kAcc) & 1))) {
                atomicOr(w.status, kStatusTimeout);
                abort_sh = 1;
            }
            if (__any_sync(0xffffffffu, abort_sh != 0)) break;   // warp-uniform: tcgen05.ld below is collective
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // the stage (node ids, b, membership) is complete: its full barrier has fired
            mbar_wait(smem_u32(&bar_full[st]), (uint32_t)((i / kStages) & 1));
            int jv[kNodes];
            uint32_t member = 0;
#pragma unroll
            for (int nl = 0; nl < kNodes; ++nl) {
                jv[nl] = sJ[st * kNodes + nl];
                const int ms = runs ? (nl & ~3) : nl;   // a run's nodes share their parent's row
                const bool mb = jv[nl] >= 0 && (top || ((sMask[(st * kNodes + ms) * kLW + (row >> 5)] >> lane) & 1u));
                member |= (mb ? 1u : 0u) << nl;
            }
            const float4* bv4 = reinterpret_cast<const float4*>(sBv + st * kTileN);
            float best[kNodes];
#pragma unroll
            for (int pr = 0; pr < kNodes / 2; ++pr) {
                float v[32];
                tmem_ld32(tmem + tlane + (uint32_t)(slot * kTileN + pr * 2 * kR), v);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // s D + b_r as packed fp32x2 fused multiply-adds (two records per
                    // instruction, the same rounding as one FMA each), then the maximum
                    float bb = -INFINITY;
                    const float2 s2 = make_float2(scale, scale);
#pragma unroll
                    for (int r4 = 0; r4 < kR / 4; ++r4) {
                        const float4 bq = bv4[(pr * 2 + h) * (kR / 4) + r4];
                        const float2 e0 = __ffma2_rn(s2, make_float2(v[h * kR + 4 * r4 + 0], v[h * kR + 4 * r4 + 1]),
                                                     make_float2(bq.x, bq.y));
                        const float2 e1 = __ffma2_rn(s2, make_float2(v[h * kR + 4 * r4 + 2], v[h * kR + 4 * r4 + 3]),
                                                     make_float2(bq.z, bq.w));
                        bb = fmaxf(bb, fmaxf(fmaxf(e0.x, e0.y), fmaxf(e1.x, e1.y)));
                    }
                    best[pr * 2 + h] = bb;
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(smem_u32(&bar_acc_empty[slot]));
            mbar_arrive(smem_u32(&bar_empty[st]));
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
                // candidate order: tile i holds candidates k0 .. k0 + 7 (rows padded past nc)
                float4* dst = reinterpret_cast<float4*>(ex + (blockIdx.x + i * gridDim.x) * kNodes);
#pragma unroll
                for (int q4 = 0; q4 < kNodes / 4; ++q4)
                    dst[q4] = make_float4(best[4 * q4], best[4 * q4 + 1], best[4 * q4 + 2], best[4 * q4 + 3]);
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
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols));
}

template <int D, int LT, bool BF>
cudaError_t launch_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st, int pairs) {
    int nb = sm_count() / max(1, pairs * b.n_groups);
    nb = nb < 1 ? 1 : nb;
    dim3 grid(nb, pairs, b.n_groups);
    const size_t smem = score_tc_smem_lt(D, LT, BF ? 1 : 2);
    cudaFuncSetAttribute(k_score_tc<D, LT, BF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_score_tc<D, LT, BF><<<grid, 64 + 128 * LT, smem, st>>>(b, w, it, scale);
    return cudaGetLastError();
}

template <int LT, bool BF>
cudaError_t launch_tc_d(const Batch& b, const Work& w, int it, float scale, cudaStream_t st, int pairs) {
    return b.d == 128 ? launch_tc<128, LT, BF>(b, w, it, scale, st, pairs) : launch_tc<64, LT, BF>(b, w, it, scale, st, pairs);
}

}  // namespace

size_t score_tc_smem_lt(int d, int lt, int planes) {
    return (size_t)kStages * planes * (d / 64) * kTileN * 128 + (size_t)kStages * kTileN * 4 +
           (size_t)kStages * kNodes * 4 * lt * 4 + (size_t)kStages * kNodes * 4 + 1024;
}

cudaError_t launch_member(const Batch& b, const Work& w, int it, int mode, cudaStream_t st) {
    ProfScope ps_("k_member", st);
    const int lwg = (b.n_gl + 255) / 256;             // groups of 8 lane words
    int nbx = (int)((w.ms + 255) / 256);
    const int cap = (sm_count() * 8) / max(1, lwg * b.n_groups);
    nbx = nbx < 1 ? 1 : (nbx > cap ? (cap < 1 ? 1 : cap) : nbx);
    k_member<<<dim3(nbx, lwg, b.n_groups), 256, 0, st>>>(b, w, it, mode);
    return cudaGetLastError();
}

cudaError_t launch_score_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st) {
    if (it > 0) {
        // membership words of the group's union parents (the level above the scored one)
        const cudaError_t e = launch_member(b, w, it, 0, st);
        if (e != cudaSuccess) return e;
    }
    ProfScope ps_("k_score_tc", st);
    const int lane_tiles = (b.n_gl + kTileM - 1) / kTileM;
    const bool bf = b.fmt == kFmtBf16;
    if (lane_tiles >= 2) {
        const int pairs = (lane_tiles + 1) / 2;
        return bf ? launch_tc_d<2, true>(b, w, it, scale, st, pairs) : launch_tc_d<2, false>(b, w, it, scale, st, pairs);
    }
    return bf ? launch_tc_d<1, true>(b, w, it, scale, st, 1) : launch_tc_d<1, false>(b, w, it, scale, st, 1);
}

}  // namespace zha
