// zha_attn.cu - exact attention over the routed token set (split-KV flash-decode).
//
// What is computed (pages: fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的 —
// exact attention only over the raw rows that routing kept; wqu.guru, section "How does top-p
// routing pick tokens?" — token 0 attended as a sink every time): for lane x,
//     A_x = {0} U {tokens of the level-1 chunks kept by x} U [T C^L, N)
//     o_x = sum_{t in A_x} exp(s q.k_t - M) v_t / sum_{t in A_x} exp(s q.k_t - M).
//
// Work layout: each (sequence, KV head) group owns a list of segments of C positions -
// the sink segment (only position 0 valid), the union of its lanes' kept chunks (a lane
// attends a chunk only if it kept it; token 0 is left to the sink), then the tail in
// pieces of C (positions >= N invalid).  A block handles one split of consecutive
// segments for 8*WB lanes of the group: K/V rows of 32 positions at a time are staged
// in shared memory and read by every warp; each warp keeps an online softmax (max, sum,
// o[]) for its 8 lanes.  k_combine merges the splits of each lane.
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kTile = 32;

template <int D>
__global__ void __launch_bounds__(256) k_attn(Batch b, Work w, float scale) {
    constexpr int RS = D + 8;                    // padded shared row (bf16)
    constexpr int PR = D + 4;                    // partial record (f32): o[D], max, sum
    __shared__ __align__(16) __nv_bfloat16 sK[kTile * RS];
    __shared__ __align__(16) __nv_bfloat16 sV[kTile * RS];
    __shared__ int64_t s_tok[kTile];
    __shared__ int32_t s_cid[kTile];

    const int grp = blockIdx.z;
    const int s = grp / b.Hkv, g = grp % b.Hkv;
    const SeqDev& sq = b.seqs[s];
    const int WB = min(8, (b.n_gl + 7) / 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int y = (blockIdx.y * WB + warp) * 8 + (lane >> 2);
    const int q = lane & 3;
    const bool lane_ok = y < b.n_gl;
    const int64_t x = lane_of(b, s, g, lane_ok ? y : 0);

    const int64_t C = sq.C;
    const int64_t T = sq.T, N = sq.N;
    const int64_t tail0 = T * sq.top;
    const int64_t tail = N - tail0;
    const int has_sink = seq_has_sink(sq);
    const int64_t nu = T >= 1 ? (int64_t)w.ucount[grp] : 0;
    const int64_t nseg = has_sink + nu + (tail + C - 1) / C;
    const int64_t SEGS = batch_segs(b, (int)C);
    const int64_t split = blockIdx.x;
    const int64_t sg0 = split * SEGS;
    if (sg0 >= nseg) return;
    const int64_t sg1 = min(nseg, sg0 + SEGS);
    const int64_t npos = (sg1 - sg0) * C;

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
    float o[D / 4];
#pragma unroll
    for (int k = 0; k < D / 4; ++k) o[k] = 0.0f;
    float mx = -INFINITY, lsum = 0.0f;

    const uint32_t* kb1 = w.kept[1] + x * w.W[1];
    const int32_t* ul = w.ulist + (int64_t)grp * w.us;
    const __nv_bfloat16* Kg = sq.K + (int64_t)g * sq.ld * D;
    const __nv_bfloat16* Vg = sq.V + (int64_t)g * sq.ld * D;

    for (int64_t p0 = 0; p0 < npos; p0 += kTile) {
        __syncthreads();
        if (threadIdx.x < kTile) {
            const int64_t pp = p0 + threadIdx.x;
            int64_t tok = -1;
            int32_t cid = -1;
            if (pp < npos) {
                const int64_t seg = sg0 + pp / C, off = pp % C;
                if (has_sink && seg == 0) {
                    tok = off == 0 ? 0 : -1;
                } else {
                    const int64_t k = seg - has_sink;
                    if (k < nu) {
                        const int64_t j = ul[k];
                        const int64_t t = j * C + off;
                        tok = (t == 0 && has_sink) ? -1 : t;
                        cid = (int32_t)j;
                    } else {
                        const int64_t t = tail0 + (k - nu) * C + off;
                        tok = t < N ? t : -1;
                    }
                }
            }
            s_tok[threadIdx.x] = tok;
            s_cid[threadIdx.x] = cid;
        }
        __syncthreads();
        constexpr int PIECES = D / 8;            // 16-byte pieces per row
        for (int i = threadIdx.x; i < kTile * PIECES; i += blockDim.x) {
            const int rr = i / PIECES, c = i % PIECES;
            const int64_t t = s_tok[rr];
            uint4 vk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (t >= 0) {
                vk = __ldg(reinterpret_cast<const uint4*>(Kg + t * D) + c);
                vv = __ldg(reinterpret_cast<const uint4*>(Vg + t * D) + c);
            }
            *reinterpret_cast<uint4*>(sK + rr * RS + c * 8) = vk;
            *reinterpret_cast<uint4*>(sV + rr * RS + c * 8) = vv;
        }
        __syncthreads();

        float sc[kTile];
        float tmax = -INFINITY;
#pragma unroll
        for (int tt = 0; tt < kTile; ++tt) {
            const uint2* row = reinterpret_cast<const uint2*>(sK + tt * RS);
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                const uint2 u = row[4 * i + q];
                const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                dot = fmaf(qv[4 * i], a0.x, dot);
                dot = fmaf(qv[4 * i + 1], a0.y, dot);
                dot = fmaf(qv[4 * i + 2], a1.x, dot);
                dot = fmaf(qv[4 * i + 3], a1.y, dot);
            }
            dot += __shfl_xor_sync(kFull, dot, 1);
            dot += __shfl_xor_sync(kFull, dot, 2);
            const int64_t t = s_tok[tt];
            const int32_t cid = s_cid[tt];
            bool member = t >= 0;
            if (member && cid >= 0) member = (__ldg(kb1 + (cid >> 5)) >> (cid & 31)) & 1u;
            sc[tt] = member ? scale * dot : -INFINITY;
            tmax = fmaxf(tmax, sc[tt]);
        }
        if (tmax > -INFINITY) {
            const float mn = fmaxf(mx, tmax);
            const float c = expf(mx - mn);
            lsum *= c;
#pragma unroll
            for (int k = 0; k < D / 4; ++k) o[k] *= c;
            mx = mn;
#pragma unroll
            for (int tt = 0; tt < kTile; ++tt) {
                if (sc[tt] > -INFINITY) {
                    const float wgt = expf(sc[tt] - mx);
                    lsum += wgt;
                    const uint2* row = reinterpret_cast<const uint2*>(sV + tt * RS);
#pragma unroll
                    for (int i = 0; i < D / 16; ++i) {
                        const uint2 u = row[4 * i + q];
                        const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                        const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                        o[4 * i] = fmaf(wgt, a0.x, o[4 * i]);
                        o[4 * i + 1] = fmaf(wgt, a0.y, o[4 * i + 1]);
                        o[4 * i + 2] = fmaf(wgt, a1.x, o[4 * i + 2]);
                        o[4 * i + 3] = fmaf(wgt, a1.y, o[4 * i + 3]);
                    }
                }
            }
        }
    }
    if (lane_ok) {
        float* pp = w.part + (x * w.s_cap + split) * PR;
        float4* po = reinterpret_cast<float4*>(pp);
#pragma unroll
        for (int i = 0; i < D / 16; ++i) po[4 * i + q] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        if (q == 0) {
            pp[D] = mx;
            pp[D + 1] = lsum;
        }
    }
}

// out[x] = sum_splits exp(m_s - M) o_s / sum_splits exp(m_s - M) l_s.
// One block of kCombThreads per lane: the splits' maximum M by a block reduction, then warp
// w sums splits w, w + 8, ... (each thread D/32 dims) and the warps' sums are added in warp
// order, so the result does not depend on scheduling.
constexpr int kCombThreads = 256;

// Sum of the warps' weighted denominators, in the order the output's division uses.
__device__ __forceinline__ float dd_all(const float* s_den, int nw) {
    float dd = 0.0f;
    for (int i = 0; i < nw; ++i) dd += s_den[i];
    return dd;
}

template <int D>
__global__ void __launch_bounds__(kCombThreads) k_combine(Batch b, Work w, float* out) {
    constexpr int PR = D + 4;
    constexpr int NW = kCombThreads / 32;
    constexpr int DPT = D / 32;                  // dims per thread
    __shared__ float s_red[NW];
    __shared__ __align__(16) float s_num[NW][D];
    __shared__ float s_den[NW];
    const int64_t x = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = (int)(x / ((int64_t)b.n_q * b.Hq));
    const int h = (int)(x % b.Hq);
    const int g = h / b.G;
    const int grp = s * b.Hkv + g;
    const SeqDev& sq = b.seqs[s];
    const int64_t C = sq.C, T = sq.T;
    const int64_t tail = sq.N - T * sq.top;
    const int has_sink = seq_has_sink(sq);
    const int64_t nu = T >= 1 ? (int64_t)w.ucount[grp] : 0;
    const int64_t nseg = has_sink + nu + (tail + C - 1) / C;
    const int64_t SEGS = batch_segs(b, (int)C);
    const int64_t nsplit = (nseg + SEGS - 1) / SEGS;
    const float* pp = w.part + x * w.s_cap * PR;
    float M = -INFINITY;
    for (int64_t sp = tid; sp < nsplit; sp += kCombThreads)
        if (pp[sp * PR + D + 1] > 0.0f) M = fmaxf(M, pp[sp * PR + D]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) s_red[warp] = M;
    __syncthreads();
    M = s_red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) M = fmaxf(M, s_red[i]);
    float num[DPT];
#pragma unroll
    for (int k = 0; k < DPT; ++k) num[k] = 0.0f;
    float den = 0.0f;
    for (int64_t sp = warp; sp < nsplit; sp += NW) {
        const float* rec = pp + sp * PR;
        const float l = rec[D + 1];
        if (l > 0.0f) {
            const float c = expf(rec[D] - M);
            if constexpr (DPT == 4) {
                const float4 o4 = reinterpret_cast<const float4*>(rec)[lane];
                num[0] = fmaf(c, o4.x, num[0]);
                num[1] = fmaf(c, o4.y, num[1]);
                num[2] = fmaf(c, o4.z, num[2]);
                num[3] = fmaf(c, o4.w, num[3]);
            } else {
#pragma unroll
                for (int k = 0; k < DPT; ++k) num[k] = fmaf(c, rec[lane * DPT + k], num[k]);
            }
            den = fmaf(c, l, den);
        }
    }
#pragma unroll
    for (int k = 0; k < DPT; ++k) s_num[warp][lane * DPT + k] = num[k];
    if (lane == 0) s_den[warp] = den;
    __syncthreads();
    if (tid < D) {
        float nn = 0.0f, dd = 0.0f;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            nn += s_num[i][tid];
            dd += s_den[i];
        }
        // a lane with no attended token (possible only on one shard of a sharded sequence)
        // gets 0 and a log-sum-exp of -inf, so that the ranks' combine ignores it
        out[x * D + tid] = dd > 0.0f ? nn / dd : 0.0f;
    }
    if (tid == 0) {
        if (w.lse_out) w.lse_out[x] = dd_all(s_den, NW) > 0.0f ? M + logf(dd_all(s_den, NW)) : -INFINITY;
        int64_t a = tail;
        if (T >= 1) {
            a += (int64_t)w.kcount[(int64_t)1 * w.lanes_cap + x] * C;
            if (has_sink) {
                const uint32_t first = w.kept[1][x * w.W[1]];
                a += 1 - (int64_t)(first & 1u);
            }
        }
        atomicAdd(&w.ctr[kCtrLaneTokens], (unsigned long long)a);
    }
}

}  // namespace

cudaError_t launch_attn(const Batch& b, const Work& w, int64_t max_splits, float scale, cudaStream_t st) {
    if (max_splits <= 0) return cudaSuccess;
    // the tensor-core kernel's grid holds the splits in y (at most 65,535: caches of up to
    // ~268M tokens); longer caches use the CUDA-core kernel
    if (attn_on_tensor_cores(b) && max_splits <= 65535)
        return launch_attn_tc(b, w, max_splits, scale, st);
    const int WB = min(8, (b.n_gl + 7) / 8);
    const int lane_blocks = (b.n_gl + 8 * WB - 1) / (8 * WB);
    dim3 grid((unsigned)max_splits, lane_blocks, b.n_groups);
    ProfScope ps_("k_attn", st);
    if (b.d == 128)
        k_attn<128><<<grid, 32 * WB, 0, st>>>(b, w, scale);
    else
        k_attn<64><<<grid, 32 * WB, 0, st>>>(b, w, scale);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Batch& b, const Work& w, float* out, cudaStream_t st) {
    ProfScope ps_("k_combine", st);
    if (b.d == 128)
        k_combine<128><<<b.n_lanes, kCombThreads, 0, st>>>(b, w, out);
    else
        k_combine<64><<<b.n_lanes, kCombThreads, 0, st>>>(b, w, out);
    return cudaGetLastError();
}

}  // namespace zha
