// zha_attn_tc.cu - exact attention over the routed token set on the tcgen05 tensor cores.
//
// Same result as k_attn (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的 —
// 只对少量保留下来的原始 KV 条目做精确注意力; wqu.guru, section "How does top-p routing pick
// tokens?" — token 0 is always attended): for every lane x of a (sequence, KV head) group,
//     o_x = sum_{t in A_x} exp(s q.k_t - M) v_t / sum_{t in A_x} exp(s q.k_t - M),
// A_x = {0} U tokens of the level-1 chunks x kept U tail.  Used when a group holds many
// lanes, so that a tile of 128 lanes x 128 token positions is a dense contraction:
//   S = Q K^T      tcgen05.mma kind::f16 (bf16 x bf16 products are exact, f32 accumulate)
//   P = exp(s S - m) on the lanes' own positions (0 elsewhere), split P = P_hi + P_lo (bf16)
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
constexpr int kPos = 128;       // token positions per tile (MMA N of QK^T, K of PV)
constexpr int kThreads = 256;
constexpr float kLazy = 8.0f;   // raise the running max only when exceeded by this much
constexpr uint64_t kWaitNs = 2000000000ull;   // bound on any wait for the tensor pipeline
constexpr int kBlock = kRows * 128;   // bytes of one 128-byte-wide block of 128 rows

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

// Offset of 16-byte chunk c16 (8 bf16) of row r in a K-major tile of 128-byte blocks.
__device__ __forceinline__ uint32_t kmaj(int r, int c16) {
    return (uint32_t)((c16 >> 3) * kBlock + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}
// Offset of 16-byte chunk c16 (8 bf16 along d) of token row t in the MN-major V tile.
__device__ __forceinline__ uint32_t mnmaj(int t, int c16) {
    return (uint32_t)((c16 >> 3) * kBlock + (t >> 3) * 1024 + (t & 7) * 128 + (((c16 & 7) ^ (t & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(Batch b, Work w, float scale) {
    constexpr int KBD = D / 64;                 // 128-byte blocks along d (bf16)
    constexpr int PR = D + 4;
    constexpr int TCOLS = 256;                  // S: columns [0,128), O: [128, 128+D)
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    unsigned char* sQ = base;                               // KBD blocks
    unsigned char* sK = sQ + KBD * kBlock;                  // KBD blocks
    unsigned char* sV0 = sK + KBD * kBlock;                 // 2 x KBD blocks (MN-major, double buffer)
    unsigned char* sPh = sV0 + 2 * KBD * kBlock;            // 2 blocks
    unsigned char* sPl = sPh + 2 * kBlock;                  // 2 blocks
    int32_t* s_tok0 = reinterpret_cast<int32_t*>(sPl + 2 * kBlock);  // [2][kPos]
    int32_t* s_cid0 = s_tok0 + 2 * kPos;                             // [2][kPos]
    uint32_t* s_mem0 = reinterpret_cast<uint32_t*>(s_cid0 + 2 * kPos);  // [2][kRows][kPos/32] lane masks
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_sh;

    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int64_t C = sq.C, T = sq.T, N = sq.N;
    const int64_t tail0 = T * sq.top;
    const int64_t tail = N - tail0;
    const int has_sink = T >= 1 ? 1 : 0;
    const int64_t nu = has_sink ? (int64_t)w.ucount[grp] : 0;
    const int64_t nseg = has_sink + nu + (tail + C - 1) / C;
    const int64_t SEGS = segs_per_split(b.n_gl, (int)C);
    const int64_t split = blockIdx.x;
    const int64_t sg0 = split * SEGS;
    if (sg0 >= nseg) return;
    const int64_t npos = (min(nseg, sg0 + SEGS) - sg0) * C;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int y0 = blockIdx.y * kRows;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tmem_sh)), "r"(TCOLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&mbar)));
        asm volatile("fence.mbarrier_init.release.cluster;");
        abort_sh = 0;
    }
    // Q tile: 128 lane rows of the group (zero past the group's lanes).
    for (int i = tid; i < kRows * (D / 8); i += kThreads) {
        const int r = i / (D / 8), c16 = i % (D / 8);
        const int y = y0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (y < b.n_gl) v = __ldg(reinterpret_cast<const uint4*>(b.Q + lane_of(b, s, g, y) * D) + c16);
        *reinterpret_cast<uint4*>(sQ + kmaj(r, c16)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_sh;
    const uint32_t tS = tmem, tO = tmem + 128;

    // Softmax state of lane row `tid` (threads 0..127; warp w reads TMEM lanes 32w..32w+31).
    const int row = tid & 127;
    const int y = y0 + row;
    const bool y_ok = y < b.n_gl;                  // lane row `row` is one of the group's lanes
    const bool row_ok = tid < kRows && y_ok;      // ... and this thread runs its softmax
    const int64_t x = lane_of(b, s, g, y < b.n_gl ? y : 0);
    const uint32_t* kb1 = w.kept[1] + x * w.W[1];
    const uint32_t lane_t = (uint32_t)((warp & 3) * 32) << 16;
    float m_ref = -INFINITY, lsum = 0.0f;

    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    const __nv_bfloat16* Kg = sq.K + (int64_t)g * sq.ld * D;
    const __nv_bfloat16* Vg = sq.V + (int64_t)g * sq.ld * D;
    uint32_t phase = 0;
    bool first_pv = true;

    // Token of each position of tile p0 into buffer `st`: sink segment (position 0 only),
    // kept chunks, tail.  cid -2: no token, -1: every lane, >= 0: chunk id.
    auto resolve = [&](int64_t p0, int st) {
        if (tid < kPos) {
            const int64_t pp = p0 + tid;
            int32_t tok = -1, cid = -2;
            if (pp < npos) {
                const int64_t seg = sg0 + pp / C, off = pp % C;
                if (has_sink && seg == 0) {
                    if (off == 0) { tok = 0; cid = -1; }
                } else {
                    const int64_t k = seg - has_sink;
                    if (k < nu) {
                        const int64_t j = ul[k];
                        const int64_t t = j * C + off;
                        if (t != 0) { tok = (int32_t)t; cid = (int32_t)j; }
                    } else {
                        const int64_t t = tail0 + (k - nu) * C + off;
                        if (t < N) { tok = (int32_t)t; cid = -1; }
                    }
                }
            }
            s_tok0[st * kPos + tid] = tok;
            s_cid0[st * kPos + tid] = cid;
        }
    };
    // Asynchronous gather of the K (K-major) and V (MN-major) rows of buffer st's tokens;
    // empty positions are zero-filled.
    auto issue_kv = [&](int st, bool with_k) {
        for (int i = tid; i < kPos * (D / 8); i += kThreads) {
            const int t = i / (D / 8), c16 = i % (D / 8);
            const int32_t tok = s_tok0[st * kPos + t];
            const uint32_t n = tok >= 0 ? 16u : 0u;
            const int64_t row = tok >= 0 ? tok : 0;
            const void* gk = reinterpret_cast<const uint4*>(Kg + row * D) + c16;
            const void* gv = reinterpret_cast<const uint4*>(Vg + row * D) + c16;
            if (with_k)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(sK + kmaj(t, c16))), "l"(gk), "r"(n) : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(sV0 + st * KBD * kBlock + mnmaj(t, c16))),
                         "l"(gv), "r"(n) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // Membership masks of tile p0 (buffer bs) for lane row `row`: position pp is attended
    // by the lane iff it holds a token and its segment is the sink, the tail, or a chunk
    // the lane kept.  Run by warps 4-7 (one lane row per thread) ahead of the softmax.
    auto build_mem = [&](int64_t p0, int bs) {
        uint32_t mw[kPos / 32];
#pragma unroll
        for (int k = 0; k < kPos / 32; ++k) mw[k] = 0;
        const int64_t segA = p0 / C;
        const int64_t segB = min((p0 + kPos - 1) / C, nseg - sg0 - 1);
        for (int64_t sr = segA; sr <= segB; sr += 8) {
            uint32_t lb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t seg = sg0 + sr + i;
                uint32_t bit = 0;
                if (sr + i <= segB) {
                    if (has_sink && seg == 0) {
                        bit = 1;
                    } else {
                        const int64_t k = seg - has_sink;
                        if (k < nu) {
                            const int32_t j = __ldg(ul + k);
                            bit = (__ldg(kb1 + (j >> 5)) >> (j & 31)) & 1u;
                        } else {
                            bit = 1;
                        }
                    }
                }
                lb[i] = bit;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (!lb[i]) continue;
                const int64_t a = max((int64_t)0, (sr + i) * C - p0);
                const int64_t e = min((int64_t)kPos, (sr + i + 1) * C - p0);
                for (int64_t pp = a; pp < e; ++pp) mw[pp >> 5] |= 1u << (pp & 31);
            }
        }
        const int32_t* tk = s_tok0 + bs * kPos;
#pragma unroll
        for (int k = 0; k < kPos / 32; ++k) {
            uint32_t valid = 0;
            for (int i = 0; i < 32; ++i) valid |= (tk[k * 32 + i] >= 0 ? 1u : 0u) << i;
            s_mem0[(bs * kRows + row) * (kPos / 32) + k] = y_ok ? (mw[k] & valid) : 0u;
        }
    };

    resolve(0, 0);
    __syncthreads();
    if (warp >= 4) build_mem(0, 0);
    issue_kv(0, true);
    int st = 0;
    for (int64_t p0 = 0; p0 < npos; p0 += kPos, st ^= 1) {
        const bool more = p0 + kPos < npos;
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (tid == 0) {
            const uint32_t q0 = su32(sQ), k0 = su32(sK);
#pragma unroll
            for (int kb = 0; kb < KBD; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t off = kb * kBlock + kk * 32;
                    mma_bf16(tS, desc_sw128(q0 + off, 16, 1024), desc_sw128(k0 + off, 16, 1024),
                             idesc_bf16(kPos, 0), (kb | kk) ? 1u : 0u);
                }
            commit(su32(&mbar));
        }
        __syncwarp();
        if (more) resolve(p0 + kPos, st ^ 1);
        if (!wait_phase(su32(&mbar), phase) && lane == 0) {
            atomicOr(w.status, kStatusTimeout);
            abort_sh = 1;
        }
        phase ^= 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        __syncthreads();                       // next tile's tokens visible; K buffer free
        if (more) issue_kv(st ^ 1, true);      // overlaps this tile's softmax and P V

        // warps 4-7: next tile's membership masks; warps 0-3: softmax of this tile
        if (warp >= 4) {
            if (more) build_mem(p0 + kPos, st ^ 1);
        } else {
            uint32_t mem[kPos / 32];
#pragma unroll
            for (int k = 0; k < kPos / 32; ++k) mem[k] = s_mem0[(st * kRows + row) * (kPos / 32) + k];
            float tmax = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < kPos / 16; ++c) {
                float v[16];
                tld16(tS + lane_t + c * 16, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int pp = c * 16 + i;
                    if ((mem[pp >> 5] >> (pp & 31)) & 1u) tmax = fmaxf(tmax, scale * v[i]);
                }
            }
            if (!row_ok) tmax = -INFINITY;
            // Raise this lane's reference max if the tile exceeds it by more than kLazy.
            // The O rescale reads and writes tensor memory with warp-collective
            // instructions, so the whole warp runs it (factor 1 on lanes that keep theirs).
            const bool need = tmax > -INFINITY && m_ref > -INFINITY && tmax > m_ref + kLazy;
            const float f = need ? expf(m_ref - tmax) : 1.0f;
            if (tmax > -INFINITY && m_ref == -INFINITY) m_ref = tmax;
            if (need) {
                lsum *= f;
                m_ref = tmax;
            }
            if (__any_sync(0xffffffffu, need) && !first_pv) {
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    float o[16];
                    tld16(tO + lane_t + c * 16, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] *= f;
                    tst16(tO + lane_t + c * 16, o);
                }
            }
            // warps read/write TMEM uniformly; rows without members write zero P
#pragma unroll 1
            for (int c = 0; c < kPos / 16; ++c) {
                float v[16];
                tld16(tS + lane_t + c * 16, v);
                uint32_t hi[8], lo[8];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const int pp = c * 16 + i;
                    float p0v = 0.0f, p1v = 0.0f;
                    if (row_ok && ((mem[pp >> 5] >> (pp & 31)) & 1u)) p0v = expf(fmaf(scale, v[i], -m_ref));
                    if (row_ok && ((mem[(pp + 1) >> 5] >> ((pp + 1) & 31)) & 1u)) p1v = expf(fmaf(scale, v[i + 1], -m_ref));
                    lsum += p0v;
                    lsum += p1v;
                    const __nv_bfloat162 h = __floats2bfloat162_rn(p0v, p1v);
                    const float2 hf = __bfloat1622float2(h);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0v - hf.x, p1v - hf.y);
                    hi[i / 2] = *reinterpret_cast<const uint32_t*>(&h);
                    lo[i / 2] = *reinterpret_cast<const uint32_t*>(&l2);
                }
                // positions c*16 .. c*16+15 are 16-byte chunks 2c and 2c+1 of this row
                *reinterpret_cast<uint4*>(sPh + kmaj(row, 2 * c)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sPh + kmaj(row, 2 * c + 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
                *reinterpret_cast<uint4*>(sPl + kmaj(row, 2 * c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4*>(sPl + kmaj(row, 2 * c + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (tid == 0) {
            const uint32_t v0 = su32(sV0 + st * KBD * kBlock);
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                const uint32_t a0 = su32(pass == 0 ? sPh : sPl);
#pragma unroll
                for (int ks = 0; ks < kPos / 16; ++ks) {
                    // A: K-major P, 16 positions = 32 bytes; B: MN-major V, 16 tokens = 2 atoms
                    const uint32_t aoff = (ks >> 2) * kBlock + (ks & 3) * 32;
                    const uint32_t boff = ks * 2048;
                    mma_bf16(tO, desc_sw128(a0 + aoff, 16, 1024), desc_sw128(v0 + boff, kBlock, 1024),
                             idesc_bf16(D, 1), (first_pv && pass == 0 && ks == 0) ? 0u : 1u);
                }
            }
            commit(su32(&mbar));
        }
        __syncwarp();
        if (!wait_phase(su32(&mbar), phase) && lane == 0) {
            atomicOr(w.status, kStatusTimeout);
            abort_sh = 1;
        }
        phase ^= 1;
        first_pv = false;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        __syncthreads();
        if (abort_sh) break;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // partial (o, m, l) of every lane row of the tile
    if (warp < 4) {
        float* pp = w.part + (x * w.s_cap + split) * PR;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            float o[16];
            tld16(tO + lane_t + c * 16, o);
            if (row_ok && !abort_sh) {
                float4* po = reinterpret_cast<float4*>(pp + c * 16);
                po[0] = make_float4(o[0], o[1], o[2], o[3]);
                po[1] = make_float4(o[4], o[5], o[6], o[7]);
                po[2] = make_float4(o[8], o[9], o[10], o[11]);
                po[3] = make_float4(o[12], o[13], o[14], o[15]);
            }
        }
        if (row_ok && !abort_sh) {
            pp[D] = m_ref;
            pp[D + 1] = lsum;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS));
}

}  // namespace

size_t attn_tc_smem(int d) {
    const int kbd = d / 64;
    return (size_t)(4 * kbd + 4) * kBlock + 4 * kPos * 4 + 2 * kRows * (kPos / 32) * 4 + 1024;
}

cudaError_t launch_attn_tc(const Batch& b, const Work& w, int64_t max_splits, float scale, cudaStream_t st) {
    if (max_splits <= 0) return cudaSuccess;
    ProfScope ps_("k_attn_tc", st);
    const int lane_tiles = (b.n_gl + kRows - 1) / kRows;
    dim3 grid((unsigned)max_splits, lane_tiles, b.n_groups);
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
