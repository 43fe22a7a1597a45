// zha_attn_tc.cu - exact attention over the routed token set on the tcgen05 tensor cores.
//
// Same result as k_attn (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的 —
// exact attention only over the raw rows that routing kept; wqu.guru, section "How does top-p
// routing pick tokens?" — token 0 is always attended): for every lane x of a (sequence, KV head) group,
//     o_x = sum_{t in A_x} exp(s q.k_t - M) v_t / sum_{t in A_x} exp(s q.k_t - M),
// A_x = {0} U tokens of the level-1 chunks x kept U tail.  Used when a group holds many
// lanes, so that a tile of 128 lanes x 128 token positions is a dense contraction:
//   S = Q K^T      tcgen05.mma kind::f16 (bf16 x bf16 products are exact, f32 accumulate)
//   P = exp(s S - m) on the lanes' own positions (0 elsewhere), split P = P_hi + P_lo (bf16,
//   each rounded to 8 significant bits by an integer add on its bits)
//   O += P_hi V + P_lo V   (P carries ~2^-17 relative error; V is exact)
// O stays in tensor memory for the whole split; the running max m is raised lazily (only
// when a tile's max exceeds it by more than 8, then O and the sum are rescaled), so most
// tiles never touch O.  Partials (o, m, l) per (lane, split) go to the same workspace as the
// CUDA-core kernel, and k_combine merges them.
//
// Shared-memory operands (all 128-byte swizzled, 16-byte chunk c of a 128-byte row r at
// c ^ (r % 8)): Q, K and P are K-major ([K block][128 rows][128 B]); V is MN-major
// ([d block of 64][16 atoms of 8 tokens][8 rows][128 B]): descriptor LBO = 16 KB between
// d blocks, SBO = 1 KB between 8-token atoms.
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr int kRows = 128;      // lanes per tile (MMA M)
constexpr int kPos = 64;        // token positions per tile (MMA N of QK^T, K of PV)
constexpr int kThreads = 256;   // 8 warps: 2 per TMEM lane quarter, each half of the positions
constexpr int kParts = kThreads / 128;
constexpr float kLazy = 8.0f;   // raise the running max only when exceeded by this much
constexpr uint64_t kWaitNs = 2000000000ull;   // bound on any wait for the tensor pipeline
constexpr int kBlock = kRows * 128;   // bytes of one 128-byte-wide block of 128 rows (Q)
constexpr int kBlockT = kPos * 128;   // the same for the tile's kPos token rows (K, V)

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 with bf16 A/B, f32 D, M = 128, N = n; b_mn selects an MN-major B operand.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

// Waits for the mbarrier phase with the given parity; gives up after about 2 s of wall time.
__device__ __forceinline__ bool wait_phase(uint32_t mbar, uint32_t parity) {
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

__device__ __forceinline__ void tld16(uint32_t taddr, float (&v)[16]) {
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

__device__ __forceinline__ void tst16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Offset of 16-byte chunk c16 (8 bf16) of row r in a K-major tile of 128-byte blocks of
// `blk` bytes (Q: 128 rows, K: kPos rows).
__device__ __forceinline__ uint32_t kmaj(int r, int c16, int blk) {
    return (uint32_t)((c16 >> 3) * blk + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}
// Offset of 16-byte chunk c16 (8 bf16 along d) of token row t in the MN-major V tile.
__device__ __forceinline__ uint32_t mnmaj(int t, int c16) {
    return (uint32_t)((c16 >> 3) * kBlockT + (t >> 3) * 1024 + (t & 7) * 128 + (((c16 & 7) ^ (t & 7)) << 4));
}

// A operand in tensor memory (the P tile), B from shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :
        : "r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

// Writes 16 consecutive 32-bit columns of this thread's tensor-memory lane (no wait).
__device__ __forceinline__ void tst16u(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// k_attn_tc (groups of at most 128 lanes).  One CTA of 256 threads per (lane tile of 128
// lanes, split, group); two CTAs share an SM (about 86 KB of shared memory and 256 tensor-memory columns each), so one CTA's
// waits are covered by the other's work.  Warp w reads TMEM lane quarter w % 4 and handles
// positions [32 (w / 4), 32 (w / 4) + 32) of a tile of 64; row group rg = warps rg, rg + 4.
// Tensor memory: S/P of tile buffers 0, 1 at columns [0, 64), [64, 128) (P over S in place:
// positions 16 j .. 16 j + 15 at columns 16 j, 8 columns of P_hi then 8 of P_lo); O at
// [128, 128 + D).
template <int D>
__global__ void __launch_bounds__(kThreads, 2) k_attn_tc(Batch b, Work w, float scale) {
    constexpr int KBD = D / 64;                 // 128-byte blocks along d (bf16)
    constexpr int PR = D + 4;
    constexpr uint32_t TCOLS = 256;
    constexpr uint32_t kColO = 128;
    constexpr int kPart = kPos / kParts;        // positions per warp of a row (32)
    constexpr int kRgPos = kPos / 4;            // positions a row group resolves and gathers (16)
    constexpr float kLog2e = 1.4426950408889634f;
    static_assert(kPart == 32, "a warp's part of a tile is one 32-bit membership word");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned start, reached by pointer arithmetic on the shared array so that every
    // pointer derived from it stays a shared-memory pointer (plain shared loads and stores)
    unsigned char* base = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sQ = base;                               // KBD blocks of 128 rows
    unsigned char* sK = sQ + KBD * kBlock;                  // KBD blocks of kPos rows (K-major)
    unsigned char* sV0 = sK + KBD * kBlockT;                // 2 x KBD blocks (MN-major, double buffer)
    int32_t* s_tok0 = reinterpret_cast<int32_t*>(sV0 + 2 * KBD * kBlockT);   // [2][kPos] token (-1: none)
    int32_t* s_slot0 = s_tok0 + 2 * kPos;                            // [2][kPos] per slot: union index, -1 all, -2 none
    uint32_t* s_mw0 = reinterpret_cast<uint32_t*>(s_slot0 + 2 * kPos);     // [2][4][kPos] lane masks: [lane word][slot]
    uint8_t* s_pslot0 = reinterpret_cast<uint8_t*>(s_mw0 + 2 * 4 * kPos);  // [2][kPos] slot of each position
    float* s_xmax = reinterpret_cast<float*>(s_pslot0 + 2 * kPos);        // [kParts][kRows] tile max per part
    float* s_xsum = s_xmax + kParts * kRows;                                // [kParts][kRows] row sums per part
    // mbS: the S = Q K^T of a tile is done; mbO: the P V of a tile is done (its V buffer free
    // again); mbDone: every MMA issued has completed.  One arrival each per completion.
    __shared__ __align__(8) uint64_t mbS, mbO, mbDone;
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_flag;
    volatile int& abort_sh = abort_flag;

    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int64_t C = sq.C, T = sq.T, N = sq.N;
    const int64_t tail0 = T * sq.top;
    const int64_t tail = N - tail0;
    const int has_sink = seq_has_sink(sq);
    const int64_t nu = T >= 1 ? (int64_t)w.ucount[grp] : 0;
    const int64_t nseg = has_sink + nu + (tail + C - 1) / C;
    const int64_t SEGS = batch_segs(b, (int)C);
    // grid (lane tiles, splits, groups): the lane tiles of one split run together, so each
    // K/V row they gather is read from DRAM once and from L2 by the others
    const int64_t split = blockIdx.y;
    const int64_t sg0 = split * SEGS;
    if (sg0 >= nseg) return;
    const int64_t npos = (min(nseg, sg0 + SEGS) - sg0) * C;
    const int nt = (int)((npos + kPos - 1) / kPos);       // tiles of this split
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y0 = blockIdx.x * kRows;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_sh)), "r"(TCOLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&mbS)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&mbO)));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&mbDone)));
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    // Q tile: 128 lane rows of the group (zero past the group's lanes).
    for (int i = tid; i < kRows * (D / 8); i += kThreads) {
        const int r = i / (D / 8), c16 = i % (D / 8);
        const int y = y0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (y < b.n_gl) v = __ldg(reinterpret_cast<const uint4*>(b.Q + lane_of(b, s, g, y) * D) + c16);
        *reinterpret_cast<uint4*>(sQ + kmaj(r, c16, kBlock)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_sh;
    const uint32_t tO = tmem + kColO;

    // Row (lane) state.  Warps w and w + 4 read the same TMEM lanes 32 (w % 4).. and share the
    // row; `part` selects positions [32 part, 32 part + 32) and O columns [D/2 part, ...).
    const int part = warp >> 2;
    const int rg = warp & 3;
    const int row = rg * 32 + lane;
    const int y = y0 + row;
    const bool y_ok = y < b.n_gl;
    const int64_t x = lane_of(b, s, g, y_ok ? y : 0);
    const uint32_t lane_t = (uint32_t)(rg * 32) << 16;
    float m_ref = -INFINITY, lsum = 0.0f;   // identical m_ref in the 2 warps of a row

    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    const __nv_bfloat16* Kg = sq.K + (int64_t)g * sq.ld * D;
    const __nv_bfloat16* Vg = sq.V + (int64_t)g * sq.ld * D;

    // Tokens of tile t into staging buffer t % 2: row group rg resolves positions
    // [16 rg, 16 rg + 16) (lanes 0..15 of warp rg): sink segment (position 0 only), kept
    // chunks, tail.  Also the slot table: slot k of the tile is the k-th segment it touches;
    // s_slot holds the segment's index in the group's union list (-1: every lane, -2: none),
    // s_mw the 32-lane membership words of the CTA's 128 lanes for that union chunk (copied
    // asynchronously, with the next committed group), s_pslot the slot of each position.
    // Positions and tokens fit 32 bits (caches hold < 2^31 rows).
    const int cs = (C & (C - 1)) == 0 ? __ffs((int)C) - 1 : -1;   // shift for power-of-two C
    const uint32_t* memb = w.memb + (int64_t)grp * w.ms * w.mwords + (int64_t)blockIdx.x * 4;
    auto resolve = [&](int t) {
        if (part == 0 && lane < kRgPos) {
            const int stg = t & 1;
            const int64_t p0 = (int64_t)t * kPos;
            const int q = kRgPos * rg + lane;                      // position in the tile
            const int pp = (int)p0 + q;
            const int segl = cs >= 0 ? (pp >> cs) : pp / (int)C;    // segment within the split
            const int off = pp - segl * (int)C;
            int32_t tok = -1, code = -2;
            if (pp < npos) {
                const int64_t seg = sg0 + segl;
                if (has_sink && seg == 0) {
                    code = -1;
                    if (off == 0) tok = 0;
                } else {
                    const int k = (int)(seg - has_sink);
                    if (k < nu) {
                        const int tk = ul[k] * (int)C + off;
                        code = k;
                        if (tk != 0 || !has_sink) tok = tk;
                    } else {
                        const int64_t tk = tail0 + (int64_t)(k - nu) * C + off;
                        code = -1;
                        if (tk < N) tok = (int32_t)tk;
                    }
                }
            }
            const int p0s = cs >= 0 ? ((int)p0 >> cs) : (int)p0 / (int)C;
            const int slot = segl - p0s;
            s_tok0[stg * kPos + q] = tok;
            s_pslot0[stg * kPos + q] = (uint8_t)slot;
            if (q == 0 || off == 0) {
                s_slot0[stg * kPos + slot] = code;
                const uint32_t* src = memb + (int64_t)(code >= 0 ? code : 0) * w.mwords;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                                     su32(s_mw0 + (stg * 4 + k) * kPos + slot)),
                                 "l"(src + k), "r"(code >= 0 ? 4u : 0u)
                                 : "memory");
            }
        }
    };
    // Asynchronous gather of tile t's K rows (K-major, the one K buffer) and V rows (MN-major,
    // buffer t % 2) for the positions row group rg resolved; empty positions are zero-filled.
    const int rt = part * 32 + lane;                               // thread within the row group
    auto gather = [&](int t) {
        const int stg = t & 1;
        unsigned char* vb = sV0 + stg * KBD * kBlockT;
        for (int i = rt; i < kRgPos * (D / 8); i += 64) {
            const int p = kRgPos * rg + i / (D / 8), c16 = i % (D / 8);
            const int32_t tok = s_tok0[stg * kPos + p];
            const uint32_t n = tok >= 0 ? 16u : 0u;
            const int64_t rw = tok >= 0 ? tok : 0;
            const void* gk = reinterpret_cast<const uint4*>(Kg + rw * D) + c16;
            const void* gv = reinterpret_cast<const uint4*>(Vg + rw * D) + c16;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(sK + kmaj(p, c16, kBlockT))),
                         "l"(gk), "r"(n) : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(vb + mnmaj(p, c16))), "l"(gv),
                         "r"(n) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // S = Q K^T of the tile whose keys sit in sK into S/P buffer t % 2 (thread 0)
    auto issue_s = [&](int t) {
        const uint32_t q0 = su32(sQ), k0 = su32(sK);
        const uint32_t dS = tmem + (uint32_t)((t & 1) * kPos);
#pragma unroll
        for (int kb = 0; kb < KBD; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(dS, desc_sw128(q0 + kb * kBlock + kk * 32, 16, 1024),
                         desc_sw128(k0 + kb * kBlockT + kk * 32, 16, 1024), idesc_bf16(kPos, 0), (kb | kk) ? 1u : 0u);
        commit(su32(&mbS));
    };
    // O += P_hi V + P_lo V of tile t (P in S/P buffer t % 2, V in buffer t % 2; thread 0)
    auto issue_pv = [&](int t) {
        const uint32_t tP = tmem + (uint32_t)((t & 1) * kPos);
        const uint32_t v0 = su32(sV0 + (t & 1) * KBD * kBlockT);
#pragma unroll
        for (int pass = 0; pass < 2; ++pass)
#pragma unroll
            for (int j = 0; j < kPos / 16; ++j)
                mma_bf16_ts(tO, tP + (uint32_t)(16 * j + 8 * pass), desc_sw128(v0 + j * 2048, kBlockT, 1024),
                            idesc_bf16(D, 1), (t == 0 && pass == 0 && j == 0) ? 0u : 1u);
        commit(su32(&mbO));
    };
    auto give_up = [&]() {
        if (lane == 0) {
            atomicOr(w.status, kStatusTimeout);
            abort_sh = 1;
        }
    };

    // Pipeline: tile t + 1's S is issued at the end of iteration t, ahead of tile t's P V, so
    // tile t + 1's softmax waits only for S; tile t's P V runs under tile t + 1's membership
    // and row maxima and is waited for before O is rescaled or its V buffer refilled.  Tile
    // t + 1's K/V are gathered during tile t's softmax.  S of tile t + 1 goes to the S/P
    // buffer of tile t - 1, whose P V has completed by then.
    resolve(0);
    __syncthreads();
    gather(0);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) issue_s(0);
    __syncwarp();
    for (int t = 0; t < nt; ++t) {
        const int stg = t & 1;
        const int64_t p0 = (int64_t)t * kPos;
        const bool more = t + 1 < nt;

        // This row's membership on its part of the tile from the staged lane masks.  When C
        // divides 32 and is at most 8 (tiles start on multiples of 64 positions) the part holds
        // 32/C whole slots, a multiple of 4: gather their bits (vector loads of the lane
        // word's slot row) and spread each over its C positions; otherwise walk the slots.
        uint32_t mem = 0;
        {
            const int hs = part * kPart;
            const int lw = row >> 5, bit = row & 31;
            const uint32_t* mrow = s_mw0 + (stg * 4 + lw) * kPos;
            const int32_t* codes = s_slot0 + stg * kPos;
            if (C <= 8 && 32 % C == 0) {               // slot rows read as 16-byte vectors
                const int ns_ = 32 / (int)C, k0 = hs / (int)C;
                uint32_t sb = 0;                       // bit k: slot k0 + k holds the row
                for (int k = 0; k < ns_; k += 4) {
                    const uint4 mv = *reinterpret_cast<const uint4*>(mrow + k0 + k);
                    const int4 cv = *reinterpret_cast<const int4*>(codes + k0 + k);
                    const uint32_t m4[4] = {mv.x, mv.y, mv.z, mv.w};
                    const int c4[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const bool in = c4[q] == -1 || (c4[q] >= 0 && ((m4[q] >> bit) & 1u));
                        sb |= (in ? 1u : 0u) << (k + q);
                    }
                }
                const uint32_t ones = (1u << C) - 1u;
                for (int k = 0; k < ns_; ++k)
                    if ((sb >> k) & 1u) mem |= ones << (k * (int)C);
            } else {
                const uint8_t* ps = s_pslot0 + stg * kPos;
                const int k0 = ps[hs], k1 = ps[hs + kPart - 1];
                // slot k spans positions [k C - o0, (k+1) C - o0) of the tile, o0 = p0 mod C
                const int o0 = (int)(p0 % C);
                for (int k = k0; k <= k1; ++k) {
                    const int32_t code = codes[k];
                    const bool in = code == -1 || (code >= 0 && ((mrow[k] >> bit) & 1u));
                    if (in) {
                        const int a = max(k * (int)C - o0, hs) - hs, e = min((k + 1) * (int)C - o0, hs + kPart) - hs;
                        const uint32_t hi_mask = e >= 32 ? ~0u : ((1u << e) - 1u);
                        mem |= hi_mask & ~((1u << a) - 1u);
                    }
                }
            }
            mem &= __ballot_sync(0xffffffffu, s_tok0[stg * kPos + hs + lane] >= 0);   // positions with a token
            if (!y_ok) mem = 0;
        }
        if (more) resolve(t + 1);
        if (!wait_phase(su32(&mbS), (uint32_t)(t & 1))) give_up();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

        // tile max over this part's member positions, combined with the row's other part
        const uint32_t tS = tmem + lane_t + (uint32_t)((t & 1) * kPos + part * kPart);
        float tmax = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kPart / 16; ++c) {
            float v[16];
            tld16(tS + c * 16, v);
            const uint32_t m16 = mem >> (c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if ((m16 >> i) & 1u) tmax = fmaxf(tmax, v[i]);
        }
        s_xmax[part * kRows + row] = tmax;
        // the previous tile's P V must be done before O is rescaled and its V buffer refilled
        if (t > 0) {
            if (!wait_phase(su32(&mbO), (uint32_t)((t - 1) & 1))) give_up();
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
        // partner maximum of the row and the next tile's tokens (resolved in this row group)
        // visible to the group
        asm volatile("bar.sync %0, 64;" ::"r"(1 + rg) : "memory");
        if (more) gather(t + 1);               // K: this tile's S is done; V: buffer (t + 1) % 2
        tmax = fmaxf(s_xmax[row], s_xmax[kRows + row]);
        tmax = tmax > -INFINITY ? scale * tmax : -INFINITY;

        // Raise the row's reference max if the tile exceeds it by more than kLazy; both warps
        // of the row take the same decision.  O is rescaled warp-collectively (factor 1 on
        // rows that keep theirs), each warp its half of the columns.
        const bool need = tmax > -INFINITY && m_ref > -INFINITY && tmax > m_ref + kLazy;
        const float f = need ? exp2f((m_ref - tmax) * kLog2e) : 1.0f;
        if (tmax > -INFINITY && m_ref == -INFINITY) m_ref = tmax;
        if (need) {
            lsum *= f;
            m_ref = tmax;
        }
        if (__any_sync(0xffffffffu, need) && t > 0) {
#pragma unroll 1
            for (int c = 0; c < D / (16 * kParts); ++c) {
                float o[16];
                const uint32_t col = tO + lane_t + part * (D / kParts) + c * 16;
                tld16(col, o);
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] *= f;
                tst16(col, o);
            }
        }
        // P = exp(s S - m) on member positions, split into bf16 hi + lo, written over S
        const float sl = scale * kLog2e, ml = m_ref * kLog2e;
#pragma unroll 1
        for (int c = 0; c < kPart / 16; ++c) {
            float v[16];
            tld16(tS + c * 16, v);
            const uint32_t m16 = mem >> (c * 16);
            uint32_t pk[16];                      // 8 columns of P_hi, then 8 of P_lo
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float2 a2 = __ffma2_rn(make_float2(sl, sl), make_float2(v[i], v[i + 1]), make_float2(-ml, -ml));
                const float e0 = ex2_approx(a2.x);
                const float e1 = ex2_approx(a2.y);
                const float p0v = ((m16 >> i) & 1u) ? e0 : 0.0f;
                const float p1v = ((m16 >> (i + 1)) & 1u) ? e1 : 0.0f;
                lsum += p0v;
                lsum += p1v;
                // bf16 hi = p rounded to 8 significant bits (integer add on the bits), lo =
                // the exact remainder rounded likewise; packed by byte permutes (even position
                // in the low half), so the split stays off the conversion unit
                const uint32_t h0 = (__float_as_uint(p0v) + 0x8000u) & 0xffff0000u;
                const uint32_t h1 = (__float_as_uint(p1v) + 0x8000u) & 0xffff0000u;
                const uint32_t l0 = __float_as_uint(p0v - __uint_as_float(h0)) + 0x8000u;
                const uint32_t l1 = __float_as_uint(p1v - __uint_as_float(h1)) + 0x8000u;
                pk[i / 2] = __byte_perm(h0, h1, 0x7632);
                pk[8 + i / 2] = __byte_perm(l0, l1, 0x7632);
            }
            tst16u(tS + c * 16, pk);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        // the next tile's K/V (gathered during this softmax) and lane masks must have landed
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (tid == 0 && !abort_sh) {
            if (more) issue_s(t + 1);
            issue_pv(t);
        }
        __syncwarp();
        if (abort_sh) break;
    }
    // every MMA issued above completes before O is read and tensor memory is released
    if (tid == 0) {
        commit(su32(&mbDone));
        if (!wait_phase(su32(&mbDone), 0)) give_up();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    s_xsum[part * kRows + row] = lsum;
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // partial (o, m, l) of every lane row of the tile: each warp writes its half of o
    {
        float* pp = w.part + (x * w.s_cap + split) * PR;
#pragma unroll 1
        for (int c = 0; c < D / (16 * kParts); ++c) {
            float o[16];
            tld16(tO + lane_t + part * (D / kParts) + c * 16, o);
            if (y_ok && !abort_sh) {
                float4* po = reinterpret_cast<float4*>(pp + part * (D / kParts) + c * 16);
                po[0] = make_float4(o[0], o[1], o[2], o[3]);
                po[1] = make_float4(o[4], o[5], o[6], o[7]);
                po[2] = make_float4(o[8], o[9], o[10], o[11]);
                po[3] = make_float4(o[12], o[13], o[14], o[15]);
            }
        }
        if (part == 0 && y_ok && !abort_sh) {
            pp[D] = m_ref;
            pp[D + 1] = s_xsum[row] + s_xsum[kRows + row];
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS));
}

// k_attn_pair (groups of more than 128 lanes).  One CTA per (pair of 128-lane tiles, split,
// group), one CTA per SM; warp roles (each synchronised with the others through mbarriers only):
//   warps 0-7   softmax: warp w owns TMEM lane quarter w % 4 of lane tile w / 4, one thread
//               per lane row, all 64 positions of a tile;
//   warps 8-9   MMA: warp 8 + L issues, for lane tile L, S = Q K^T of tile t + 1 and then
//               O += P V of tile t, each once its operands are ready (the two lane tiles
//               pipeline independently over the shared K/V stages);
//   warps 10-13 gather: thread q resolves position q % 64 of a tile and copies its K row
//               (q < 64) or V row (q >= 64) into a ring of kStages stages, kLag tiles in
//               flight per thread, plus the tile's slot table and lane masks.
// Both lane tiles read the same staged K/V rows.  Tensor memory (512 columns): lane tile L
// at 256 L: S/P buffers at [0, 64), [64, 128) (P over S in place: positions 16 j .. 16 j + 15
// at columns 16 j, 8 columns of P_hi then 8 of P_lo), O at [128, 128 + D).
constexpr int kLT = 2;                         // lane tiles per CTA
constexpr int kStages = 4;                     // K/V stages
constexpr int kLag = 2;                        // tiles a gather thread keeps in flight beyond the current one
constexpr int kSoftWarps = 4 * kLT;
constexpr int kMmaWarp = kSoftWarps;          // first MMA warp (one per lane tile)
constexpr int kGatherWarp = kMmaWarp + kLT;     // first gather warp
constexpr int kGatherWarps = 4;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kWsThreads = 32 * (kSoftWarps + kLT + kGatherWarps);
constexpr uint32_t kTCols = 512;
static_assert(kStages >= kLag + 1, "a stage is refilled only after the tile kLag + 1 behind it was consumed");
static_assert(kGatherThreads == 2 * kPos, "one gather thread per position and row kind (K or V)");

// True in one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one() {
    uint32_t is;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}\n" : "=r"(is));
    return is != 0;
}
__device__ __forceinline__ void arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
template <int D>
__global__ void __launch_bounds__(kWsThreads, 1) k_attn_pair(Batch b, Work w, float scale) {
    constexpr int KBD = D / 64;                 // 128-byte blocks along d (bf16)
    constexpr int PR = D + 4;
    constexpr uint32_t kColO = 128;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int kMW = 4 * kLT;                // lane-mask words per slot (32 lanes each)
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
    unsigned char* sQ = base;                                   // [kLT][KBD blocks of 128 rows]
    unsigned char* sK = sQ + kLT * KBD * kBlock;                // [kStages][KBD blocks of kPos rows], K-major
    unsigned char* sV = sK + kStages * KBD * kBlockT;           // [kStages][KBD blocks], MN-major
    int32_t* s_code = reinterpret_cast<int32_t*>(sV + kStages * KBD * kBlockT);   // [kStages][kPos]
    uint32_t* s_mw = reinterpret_cast<uint32_t*>(s_code + kStages * kPos);         // [kStages][kMW][kPos]
    uint32_t* s_valid = s_mw + kStages * kMW * kPos;                                // [kStages][2]
    uint8_t* s_pslot = reinterpret_cast<uint8_t*>(s_valid + kStages * 2);           // [kStages][kPos]
    // full[st]: the gather threads' copies of a stage landed (kGatherThreads arrivals);
    // empty[st]: every MMA reading the stage completed (one arrival per lane tile);
    // sfull[L][b] / pready[L][b]: S of buffer b done / its P written (128 arrivals);
    // pvb[L][b]: the P V reading buffer b (and every MMA of lane tile L before it) completed;
    // done[L]: all MMAs of lane tile L completed.
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], sfull[kLT][2], pready[kLT][2], pvb[kLT][2], done[kLT];
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_flag;
    volatile int& abort_sh = abort_flag;

    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int64_t C = sq.C, T = sq.T, N = sq.N;
    const int64_t tail0 = T * sq.top;
    const int64_t tail = N - tail0;
    const int has_sink = seq_has_sink(sq);
    const int64_t nu = T >= 1 ? (int64_t)w.ucount[grp] : 0;
    const int64_t nseg = has_sink + nu + (tail + C - 1) / C;
    const int64_t SEGS = batch_segs(b, (int)C);
    // grid (lane tile pairs, splits, groups): the pairs of one split run together, so each
    // K/V row they gather is read from DRAM once and from L2 by the others
    const int64_t split = blockIdx.y;
    const int64_t sg0 = split * SEGS;
    if (sg0 >= nseg) return;
    const int64_t npos = (min(nseg, sg0 + SEGS) - sg0) * C;
    const int nt = (int)((npos + kPos - 1) / kPos);       // tiles of this split
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y00 = blockIdx.x * (kLT * kRows);
    const int nL = min(kLT, (b.n_gl - y00 + kRows - 1) / kRows);   // lane tiles holding lanes

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_sh)), "r"(kTCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(&full[i])), "r"(kGatherThreads));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(&empty[i])), "r"(nL));
        }
        for (int L = 0; L < kLT; ++L)
            for (int i = 0; i < 2; ++i) {
                asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&sfull[L][i])));
                asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(&pready[L][i])), "r"(kRows));
                asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&pvb[L][i])));
            }
        for (int L = 0; L < kLT; ++L) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&done[L])));
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    // Q tiles: 128 lane rows each (zero past the group's lanes)
    for (int i = tid; i < kLT * kRows * (D / 8); i += kWsThreads) {
        const int r = i / (D / 8), c16 = i % (D / 8);
        const int y = y00 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (y < b.n_gl) v = __ldg(reinterpret_cast<const uint4*>(b.Q + lane_of(b, s, g, y) * D) + c16);
        *reinterpret_cast<uint4*>(sQ + (r / kRows) * KBD * kBlock + kmaj(r % kRows, c16, kBlock)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_sh;
    auto give_up = [&]() {
        atomicOr(w.status, kStatusTimeout);
        abort_sh = 1;
    };

    if (warp >= kGatherWarp) {
        // ------------------------------------------------------------------ gather
        const int q = tid - kGatherWarp * 32;
        const int p = q % kPos, half = q / kPos;      // half 0: K row and the slot table, 1: V row
        const int32_t* ul = w.ulist + (int64_t)grp * w.us;
        const __nv_bfloat16* src = (half == 0 ? sq.K : sq.V) + (int64_t)g * sq.ld * D;
        const uint32_t* memb = w.memb + (int64_t)grp * w.ms * w.mwords + (int64_t)blockIdx.x * kMW;
        const int cs = (C & (C - 1)) == 0 ? __ffs((int)C) - 1 : -1;   // shift for power-of-two C
        for (int t = 0; t < nt + kLag; ++t) {
            const int st = t % kStages;
            bool go = t < nt && !__any_sync(0xffffffffu, abort_sh != 0);
            if (go && t >= kStages) {
                if (!wait_phase(su32(&empty[st]), (uint32_t)((t / kStages - 1) & 1))) give_up();
                go = !__any_sync(0xffffffffu, abort_sh != 0);   // warp-uniform
            }
            if (go) {
                // position p of tile t: sink segment (position 0 only), kept chunks, tail;
                // slot = the tile's k-th segment; code = its union index (-1 all lanes, -2 none)
                const int64_t p0 = (int64_t)t * kPos;
                const int pp = (int)p0 + p;
                const int segl = cs >= 0 ? (pp >> cs) : pp / (int)C;
                const int off = pp - segl * (int)C;
                int32_t tok = -1, code = -2;
                if (pp < npos) {
                    const int64_t seg = sg0 + segl;
                    if (has_sink && seg == 0) {
                        code = -1;
                        if (off == 0) tok = 0;
                    } else {
                        const int k = (int)(seg - has_sink);
                        if (k < nu) {
                            const int tk = __ldg(ul + k) * (int)C + off;
                            code = k;
                            if (tk != 0 || !has_sink) tok = tk;
                        } else {
                            const int64_t tk = tail0 + (int64_t)(k - nu) * C + off;
                            code = -1;
                            if (tk < N) tok = (int32_t)tk;
                        }
                    }
                }
                if (half == 0) {
                    const int p0s = cs >= 0 ? ((int)p0 >> cs) : (int)p0 / (int)C;
                    const int slot = segl - p0s;
                    s_pslot[st * kPos + p] = (uint8_t)slot;
                    if (p == 0 || off == 0) {
                        s_code[st * kPos + slot] = code;
                        const uint32_t* msrc = memb + (int64_t)(code >= 0 ? code : 0) * w.mwords;
#pragma unroll
                        for (int k = 0; k < kMW; ++k)
                            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                                             su32(s_mw + (st * kMW + k) * kPos + slot)),
                                         "l"(msrc + k), "r"(code >= 0 ? 4u : 0u)
                                         : "memory");
                    }
                    const uint32_t vb = __ballot_sync(0xffffffffu, tok >= 0);
                    if (lane == 0) s_valid[st * 2 + (p >> 5)] = vb;
                }
                // the warp's 32 rows (positions p - lane ..), 16-byte chunks spread over the
                // lanes so that each copy instruction reads whole rows
                unsigned char* dst = (half == 0 ? sK : sV) + st * KBD * kBlockT;
                constexpr int CPR = D / 8;                 // 16-byte chunks per row
                constexpr int RPI = 32 / CPR;              // rows per copy instruction
                const int c16 = lane % CPR;
#pragma unroll
                for (int j = 0; j < CPR; ++j) {
                    const int r = RPI * j + lane / CPR;
                    const int32_t tr = __shfl_sync(0xffffffffu, tok, r);
                    const int pr = p - lane + r;
                    const uint32_t o = half == 0 ? kmaj(pr, c16, kBlockT) : mnmaj(pr, c16);
                    const uint4* row = reinterpret_cast<const uint4*>(src + (int64_t)(tr >= 0 ? tr : 0) * D);
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(dst + o)), "l"(row + c16),
                                 "r"(tr >= 0 ? 16u : 0u)
                                 : "memory");
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            if (t >= kLag) {
                // tile t - kLag's copies landed: visible to the tensor cores, then signalled
                asm volatile("cp.async.wait_group %0;" ::"n"(kLag) : "memory");
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                arrive(su32(&full[(t - kLag) % kStages]));
            }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
    } else if (warp >= kMmaWarp) {
        // ------------------------------------------------------------------ MMA
        // Lane tile L: S of tile t + 1 (its K landed; the P V that read its S/P buffer, tile
        // t - 1, completed), then the P V of tile t once its P is written; the stage of tile t
        // is released (one arrival of this lane tile) when those complete.  The whole warp
        // waits and one elected lane issues, with the operand descriptors formed once and
        // advanced by address offsets (issuing from a converged warp measured about twice as
        // fast per MMA as from a lone thread).
        const int L = warp - kMmaWarp;
        if (L < nL) {
            const uint64_t dq = desc_sw128(su32(sQ + L * KBD * kBlock), 16, 1024);
            const uint64_t dk0 = desc_sw128(su32(sK), 16, 1024);
            const uint64_t dv0 = desc_sw128(su32(sV), kBlockT, 1024);
            const uint32_t tO = tmem + (uint32_t)(L * 256) + kColO;
            constexpr uint32_t idS = idesc_bf16(kPos, 0), idO = idesc_bf16(D, 1);
            auto issue_s = [&](int t) {
                const uint64_t dk = dk0 + (uint64_t)(((t % kStages) * KBD * kBlockT) >> 4);
                const uint32_t dS = tmem + (uint32_t)(L * 256 + (t & 1) * kPos);
#pragma unroll
                for (int kb = 0; kb < KBD; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(dS, dq + (uint64_t)((kb * kBlock + kk * 32) >> 4),
                                 dk + (uint64_t)((kb * kBlockT + kk * 32) >> 4), idS, (kb | kk) ? 1u : 0u);
                commit(su32(&sfull[L][t & 1]));
            };
            bool ok = __all_sync(0xffffffffu, wait_phase(su32(&full[0]), 0u));
            if (ok) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (elect_one()) issue_s(0);
                __syncwarp();
            }
            for (int t = 0; t < nt && ok; ++t) {
                if (__any_sync(0xffffffffu, abort_sh != 0)) break;
                if (t + 1 < nt) {
                    ok = wait_phase(su32(&full[(t + 1) % kStages]), (uint32_t)(((t + 1) / kStages) & 1));
                    if (ok && t >= 1) ok = wait_phase(su32(&pvb[L][(t - 1) & 1]), (uint32_t)(((t - 1) >> 1) & 1));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (elect_one()) issue_s(t + 1);
                    __syncwarp();
                }
                ok = __all_sync(0xffffffffu, wait_phase(su32(&pready[L][t & 1]), (uint32_t)((t >> 1) & 1)));
                if (!ok) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (elect_one()) {
                    const uint32_t tP = tmem + (uint32_t)(L * 256 + (t & 1) * kPos);
                    const uint64_t dv = dv0 + (uint64_t)(((t % kStages) * KBD * kBlockT) >> 4);
#pragma unroll
                    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                        for (int j = 0; j < kPos / 16; ++j)
                            mma_bf16_ts(tO, tP + (uint32_t)(16 * j + 8 * pass), dv + (uint64_t)((j * 2048) >> 4), idO,
                                        (t == 0 && pass == 0 && j == 0) ? 0u : 1u);
                    commit(su32(&pvb[L][t & 1]));
                    commit(su32(&empty[t % kStages]));
                }
                __syncwarp();
            }
            if (!ok && lane == 0) give_up();
            // every MMA issued above completes before tensor memory is released
            if (elect_one()) commit(su32(&done[L]));
            __syncwarp();
            if (!__all_sync(0xffffffffu, wait_phase(su32(&done[L]), 0)) && lane == 0) give_up();
        }
    } else {
        // ------------------------------------------------------------------ softmax
        const int L = warp >> 2, wl = warp & 3;
        const int row = wl * 32 + lane;
        const int y = y00 + L * kRows + row;
        const bool y_ok = y < b.n_gl;
        const int64_t x = lane_of(b, s, g, y_ok ? y : 0);
        const uint32_t lane_t = (uint32_t)(wl * 32) << 16;
        const uint32_t tT = tmem + lane_t + (uint32_t)(L * 256);
        const int lw = L * 4 + wl, bit = lane;
        float m_ref = -INFINITY, lsum = 0.0f;
        if (L < nL) {
            for (int t = 0; t < nt; ++t) {
                const int st = t % kStages, bb = t & 1;
                const int64_t p0 = (int64_t)t * kPos;
                if (!wait_phase(su32(&full[st]), (uint32_t)((t / kStages) & 1))) give_up();
                if (__any_sync(0xffffffffu, abort_sh != 0)) break;
                // this row's membership over the tile's 64 positions from the staged lane masks
                // (as 2 words); C dividing 32 and at most 8: whole slots of C positions
                uint64_t mem = 0;
                {
                    const uint32_t* mrow = s_mw + (st * kMW + lw) * kPos;
                    const int32_t* codes = s_code + st * kPos;
                    if (C <= 8 && 32 % C == 0) {
                        const int ns_ = kPos / (int)C;
                        uint64_t sb = 0;                       // bit k: slot k holds the row
                        for (int k = 0; k < ns_; k += 4) {
                            const uint4 mv = *reinterpret_cast<const uint4*>(mrow + k);
                            const int4 cv = *reinterpret_cast<const int4*>(codes + k);
                            const uint32_t m4[4] = {mv.x, mv.y, mv.z, mv.w};
                            const int c4[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const bool in = c4[qq] == -1 || (c4[qq] >= 0 && ((m4[qq] >> bit) & 1u));
                                sb |= (in ? 1ull : 0ull) << (k + qq);
                            }
                        }
                        const uint64_t ones = (1ull << C) - 1ull;
                        for (int k = 0; k < ns_; ++k)
                            if ((sb >> k) & 1ull) mem |= ones << (k * (int)C);
                    } else {
                        const uint8_t* ps = s_pslot + st * kPos;
                        const int k0 = ps[0], k1 = ps[kPos - 1];
                        // slot k spans positions [k C - o0, (k+1) C - o0) of the tile, o0 = p0 mod C
                        const int o0 = (int)(p0 % C);
                        for (int k = k0; k <= k1; ++k) {
                            const int32_t code = codes[k];
                            const bool in = code == -1 || (code >= 0 && ((mrow[k] >> bit) & 1u));
                            if (!in) continue;
                            const int a = max(k * (int)C - o0, 0), e = min((k + 1) * (int)C - o0, kPos);
                            const uint64_t hi_mask = e >= 64 ? ~0ull : ((1ull << e) - 1ull);
                            mem |= hi_mask & ~((1ull << a) - 1ull);
                        }
                    }
                    mem &= *reinterpret_cast<const uint64_t*>(s_valid + st * 2);
                    if (!y_ok) mem = 0;
                }
                if (!wait_phase(su32(&sfull[L][bb]), (uint32_t)((t >> 1) & 1))) give_up();
                if (__any_sync(0xffffffffu, abort_sh != 0)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t tS = tT + (uint32_t)(bb * kPos);
                float v[kPos];
                {
                    uint32_t r[kPos];
#pragma unroll
                    for (int c = 0; c < kPos / 16; ++c)
                        asm volatile(
                            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                            : "=r"(r[16 * c + 0]), "=r"(r[16 * c + 1]), "=r"(r[16 * c + 2]), "=r"(r[16 * c + 3]),
                              "=r"(r[16 * c + 4]), "=r"(r[16 * c + 5]), "=r"(r[16 * c + 6]), "=r"(r[16 * c + 7]),
                              "=r"(r[16 * c + 8]), "=r"(r[16 * c + 9]), "=r"(r[16 * c + 10]), "=r"(r[16 * c + 11]),
                              "=r"(r[16 * c + 12]), "=r"(r[16 * c + 13]), "=r"(r[16 * c + 14]), "=r"(r[16 * c + 15])
                            : "r"(tS + 16 * c));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int i = 0; i < kPos; ++i) v[i] = __uint_as_float(r[i]);
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < kPos; ++i)
                    if ((mem >> i) & 1ull) mx[i & 3] = fmaxf(mx[i & 3], v[i]);
                float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                tmax = tmax > -INFINITY ? scale * tmax : -INFINITY;
                // raise the row's reference max if the tile exceeds it by more than kLazy: O
                // (complete up to the previous tile's P V) is rescaled warp-collectively,
                // factor 1 on rows that keep theirs
                const bool need = tmax > -INFINITY && m_ref > -INFINITY && tmax > m_ref + kLazy;
                const float f = need ? exp2f((m_ref - tmax) * kLog2e) : 1.0f;
                if (tmax > -INFINITY && m_ref == -INFINITY) m_ref = tmax;
                if (need) {
                    lsum *= f;
                    m_ref = tmax;
                }
                if (__any_sync(0xffffffffu, need) && t > 0) {
                    if (!wait_phase(su32(&pvb[L][(t - 1) & 1]), (uint32_t)(((t - 1) >> 1) & 1))) give_up();
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        float o[16];
                        const uint32_t col = tT + kColO + c * 16;
                        tld16(col, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= f;
                        tst16(col, o);
                    }
                }
                // P = exp(s S - m) on member positions, split into bf16 hi + lo, written over S
                const float sl = scale * kLog2e, ml = m_ref * kLog2e;
                float ls[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // the tile's row sum in 4 chains
#pragma unroll
                for (int c = 0; c < kPos / 16; ++c) {
                    uint32_t pk[16];                      // 8 columns of P_hi, then 8 of P_lo
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const int ii = 16 * c + i;
                        const float2 a2 =
                            __ffma2_rn(make_float2(sl, sl), make_float2(v[ii], v[ii + 1]), make_float2(-ml, -ml));
                        const float e0 = ex2_approx(a2.x);
                        const float e1 = ex2_approx(a2.y);
                        const uint32_t mw_ = (uint32_t)(mem >> ii);
                        const float p0v = (mw_ & 1u) ? e0 : 0.0f;
                        const float p1v = (mw_ & 2u) ? e1 : 0.0f;
                        ls[(i >> 1) & 3] += p0v + p1v;
                        // bf16 hi = p rounded to 8 significant bits (integer add on the bits),
                        // lo = the exact remainder rounded likewise; packed by byte permutes
                        // (even position in the low half)
                        const uint32_t h0 = (__float_as_uint(p0v) + 0x8000u) & 0xffff0000u;
                        const uint32_t h1 = (__float_as_uint(p1v) + 0x8000u) & 0xffff0000u;
                        const uint32_t l0 = __float_as_uint(p0v - __uint_as_float(h0)) + 0x8000u;
                        const uint32_t l1 = __float_as_uint(p1v - __uint_as_float(h1)) + 0x8000u;
                        pk[i / 2] = __byte_perm(h0, h1, 0x7632);
                        pk[8 + i / 2] = __byte_perm(l0, l1, 0x7632);
                    }
                    tst16u(tS + c * 16, pk);
                }
                lsum += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                arrive(su32(&pready[L][bb]));
            }
            // the lane tile's last P V (and every MMA before it) completed: O is final
            if (!__any_sync(0xffffffffu, abort_sh != 0)) {
                if (!wait_phase(su32(&pvb[L][(nt - 1) & 1]), (uint32_t)(((nt - 1) >> 1) & 1))) give_up();
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            }
            // partial (o, m, l) of this lane row
            float* pp = w.part + (x * w.s_cap + split) * PR;
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
                float o[16];
                tld16(tT + kColO + c * 16, o);
                if (y_ok && !abort_sh) {
                    float4* po = reinterpret_cast<float4*>(pp + c * 16);
                    po[0] = make_float4(o[0], o[1], o[2], o[3]);
                    po[1] = make_float4(o[4], o[5], o[6], o[7]);
                    po[2] = make_float4(o[8], o[9], o[10], o[11]);
                    po[3] = make_float4(o[12], o[13], o[14], o[15]);
                }
            }
            if (y_ok && !abort_sh) {
                pp[D] = m_ref;
                pp[D + 1] = lsum;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == kMmaWarp) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTCols));
}

}  // namespace

size_t attn_tc_smem(int d) {
    const int kbd = d / 64;
    return (size_t)kbd * kBlock + (size_t)3 * kbd * kBlockT + 2 * kPos * 4 + 2 * kPos * 4 + 2 * 4 * kPos * 4 +
           2 * kPos + 2 * kParts * kRows * 4 + 1024;
}

size_t attn_pair_smem(int d) {
    const int kbd = d / 64;
    return (size_t)kLT * kbd * kBlock + (size_t)2 * kStages * kbd * kBlockT + (size_t)kStages * kPos * 4 +
           (size_t)kStages * 4 * kLT * kPos * 4 + (size_t)kStages * 2 * 4 + (size_t)kStages * kPos + 1024;
}

cudaError_t launch_attn_tc(const Batch& b, const Work& w, int64_t max_splits, float scale, cudaStream_t st) {
    if (max_splits <= 0) return cudaSuccess;
    if (!b.dense) {
        const cudaError_t e = launch_member(b, w, 0, 1, st);   // lane masks of the kept level-1 chunks
        if (e != cudaSuccess) return e;
    }
    ProfScope ps_("k_attn_tc", st);
    // groups of more than one lane tile: two lane tiles per CTA share each staged K/V row;
    // otherwise one lane tile per CTA, two CTAs per SM (splits <= 65,535, checked by the caller)
    if (b.n_gl > kRows) {
        const int pairs = (b.n_gl + kLT * kRows - 1) / (kLT * kRows);
        dim3 grid(pairs, (unsigned)max_splits, b.n_groups);
        const size_t smem = attn_pair_smem(b.d);
        if (b.d == 128) {
            cudaFuncSetAttribute(k_attn_pair<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            k_attn_pair<128><<<grid, kWsThreads, smem, st>>>(b, w, scale);
        } else {
            cudaFuncSetAttribute(k_attn_pair<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            k_attn_pair<64><<<grid, kWsThreads, smem, st>>>(b, w, scale);
        }
        return cudaGetLastError();
    }
    const int lane_tiles = (b.n_gl + kRows - 1) / kRows;
    dim3 grid(lane_tiles, (unsigned)max_splits, b.n_groups);
    const size_t smem = attn_tc_smem(b.d);
    if (b.d == 128) {
        cudaFuncSetAttribute(k_attn_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_attn_tc<128><<<grid, kThreads, smem, st>>>(b, w, scale);
    } else {
        cudaFuncSetAttribute(k_attn_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_attn_tc<64><<<grid, kThreads, smem, st>>>(b, w, scale);
    }
    return cudaGetLastError();
}

}  // namespace zha
