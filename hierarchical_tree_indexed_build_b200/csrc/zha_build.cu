// zha_build.cu - tree build kernels (level-1 chunk summaries, level-up merges).
//
// What is computed (pages: "Zyphra ZHA 稀疏注意力…" fluxbbs.com, section 树形索引是怎么搭的;
// "Zyphra发布层级注意力ZHA…" wqu.guru, section "Building the tree"): for chunk j of KV head g
// and reference query q_r,
//     a_t = s q_r.k_t,   lse_r = log sum_t exp(a_t),   m_r = sum_t exp(a_t - lse_r) k_t,
//     b_r = lse_r - s q_r.m_r,
// and a level-l node is the online-softmax merge of its C children, i.e. the same summary
// over its C^l raw tokens.
//
// Thread mapping: a "worker" of 4R threads summarises one node; thread (r, quarter) owns
// reference query r and the dimensions {16 i + 4 quarter + c : c < 4} (interleaved so the
// four quarters of a row are 64 contiguous bytes).  The running state of a node is the
// unnormalised online softmax (mx, z, acc[]) with acc = sum_t exp(a_t - mx) k_t.
#include <math.h>

#include <algorithm>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

constexpr unsigned kFull = 0xffffffffu;

template <int D>
__device__ __forceinline__ void load_row_bf16(const __nv_bfloat16* row, int q, float (&v)[D / 4]) {
    const uint2* p = reinterpret_cast<const uint2*>(row);
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
        const uint2 u = __ldg(p + 4 * i + q);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v[4 * i + 0] = a.x;
        v[4 * i + 1] = a.y;
        v[4 * i + 2] = b.x;
        v[4 * i + 3] = b.y;
    }
}

// Sum over the 4 quarter-threads of a row.
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(kFull, v, 1);
    v += __shfl_xor_sync(kFull, v, 2);
    return v;
}

// m values of slope r held by thread quarter q (dims 16 i + 4 q + c) of a stored record.
template <int D>
__device__ __forceinline__ void load_row_m(const float* rec, int R, int r, int q, float (&v)[D / 4], int fmt) {
    if (fmt == kFmtFp4) {
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const float4 x = fp4_load4(rec, R, D, r, 16 * i + 4 * q);
            v[4 * i + 0] = x.x;
            v[4 * i + 1] = x.y;
            v[4 * i + 2] = x.z;
            v[4 * i + 3] = x.w;
        }
        return;
    }
    if (fmt == kFmtBf16) {
        const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(rec) + (int64_t)r * D;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(p + 16 * i + 4 * q));
            const float2 x = m_decode_bf16(u.x), y = m_decode_bf16(u.y);
            v[4 * i + 0] = x.x;
            v[4 * i + 1] = x.y;
            v[4 * i + 2] = y.x;
            v[4 * i + 3] = y.y;
        }
        return;
    }
    const __half* h = reinterpret_cast<const __half*>(rec);
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
        const uint2 hi = __ldg(reinterpret_cast<const uint2*>(h + (int64_t)r * D + 16 * i + 4 * q));
        const uint2 lo = __ldg(reinterpret_cast<const uint2*>(h + (int64_t)R * D + (int64_t)r * D + 16 * i + 4 * q));
        const float2 x = m_decode2(hi.x, lo.x), y = m_decode2(hi.y, lo.y);
        v[4 * i + 0] = x.x;
        v[4 * i + 1] = x.y;
        v[4 * i + 2] = y.x;
        v[4 * i + 3] = y.y;
    }
}

// Turn a running state into the stored summary of one node and write it:
// m_r = acc / z (stored in the tree's format: fp16 hi + lo planes, or one bf16 plane),
// lse_r = mx + log z, b_r = lse_r - s q_r.m_r with the stored m.  Returns lse_r; the stored m
// (decoded) is left in `m` so the parent folds exactly what a merge from the record would read.
template <int D>
__device__ __forceinline__ float finalize_store(float mx, float z, const float (&acc)[D / 4],
                                                const float (&qv)[D / 4], float scale, float* rec,
                                                float* lse, int r, int q, int R, bool store, int32_t* rflag,
                                                float (&m)[D / 4], int fmt) {
    const float inv = 1.0f / z;
    float qm = 0.0f;
    bool bad = false;
    __half* hp = reinterpret_cast<__half*>(rec);
    __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(rec);
    if (fmt == kFmtFp4) {
        // MXFP4: block k of 32 dims is held 8 dims per quarter-thread (i = 2k, 2k + 1); its
        // largest magnitude over the quad sets the scale, then every value gets its code
        uint8_t* cp = reinterpret_cast<uint8_t*>(rec);
        uint8_t* sp = cp + (int64_t)R * D / 2;
#pragma unroll
        for (int bk = 0; bk < D / kFp4Block; ++bk) {
            float a[8];
            float amax = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                a[c] = acc[8 * bk + c] * inv;
                amax = fmaxf(amax, fabsf(a[c]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
            const uint32_t E = fp4_scale_byte(amax);
            const float X = fp4_scale(E), iX = fp4_inv_scale(E);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = 2 * bk + h;
                uint32_t wv = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t code = fp4_code(a[4 * h + c] * iX);
                    wv |= code << (4 * c);
                    m[4 * i + c] = fp4_value(code, X);
                }
                if (store) *reinterpret_cast<uint16_t*>(cp + ((int64_t)r * D + 16 * i + 4 * q) / 2) = (uint16_t)wv;
            }
            if (store && q == 0) sp[(int64_t)r * (D / kFp4Block) + bk] = (uint8_t)E;
        }
#pragma unroll
        for (int k = 0; k < D / 4; ++k) qm = fmaf(qv[k], m[k], qm);
        qm = quad_sum(qm);
        const float l = mx + logf(z);
        if (store && q == 0) {
            rec[b_offset(R, D, fmt) + r] = fmaf(-scale, qm, l);
            lse[r] = l;
        }
        return l;
    }
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
        float a[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            a[c] = acc[4 * i + c] * inv;
            bad |= !(fabsf(a[c]) < 65504.0f);
        }
        if (fmt == kFmtBf16) {
            const __nv_bfloat162 b0 = __floats2bfloat162_rn(a[0], a[1]), b1 = __floats2bfloat162_rn(a[2], a[3]);
            const float2 f0 = __bfloat1622float2(b0), f1 = __bfloat1622float2(b1);
            m[4 * i] = f0.x;
            m[4 * i + 1] = f0.y;
            m[4 * i + 2] = f1.x;
            m[4 * i + 3] = f1.y;
            if (store)
                *reinterpret_cast<uint2*>(bp + (int64_t)r * D + 16 * i + 4 * q) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        } else {
            uint32_t h0, l0, h1, l1;
            m_encode2(a[0], a[1], h0, l0, m[4 * i], m[4 * i + 1]);
            m_encode2(a[2], a[3], h1, l1, m[4 * i + 2], m[4 * i + 3]);
            if (store) {
                *reinterpret_cast<uint2*>(hp + (int64_t)r * D + 16 * i + 4 * q) = make_uint2(h0, h1);
                *reinterpret_cast<uint2*>(hp + (int64_t)R * D + (int64_t)r * D + 16 * i + 4 * q) = make_uint2(l0, l1);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) qm = fmaf(qv[4 * i + c], m[4 * i + c], qm);
    }
    qm = quad_sum(qm);
    const float l = mx + logf(z);
    if (store) {
        if (q == 0) {
            rec[b_offset(R, D, fmt) + r] = fmaf(-scale, qm, l);
            lse[r] = l;
        }
        if (bad && fmt != kFmtBf16) atomicOr(rflag, 1);   // bf16 holds every finite f32 range
    }
    return l;
}

// Online-softmax merge of one child summary (lse_c, m_c) into a parent state (mx, z, acc):
// the same arithmetic, in the same order, in the streaming build and in k_merge, so a tree
// grown by appends is bit-identical to one built in one pass.
template <int D>
__device__ __forceinline__ void fold_child(float& mx, float& z, float (&acc)[D / 4], float lc,
                                           const float (&mc)[D / 4]) {
    const float mn = fmaxf(mx, lc);
    const float cp = expf(mx - mn);   // mx = -inf -> 0
    const float cc = expf(lc - mn);
    z = fmaf(z, cp, cc);
    // packed fp32x2: the same multiply and fused multiply-add per element
    const float2 cp2 = make_float2(cp, cp), cc2 = make_float2(cc, cc);
#pragma unroll
    for (int k = 0; k < D / 4; k += 2) {
        const float2 a2 = __ffma2_rn(make_float2(acc[k], acc[k + 1]), cp2, __fmul2_rn(make_float2(mc[k], mc[k + 1]), cc2));
        acc[k] = a2.x;
        acc[k + 1] = a2.y;
    }
    mx = mn;
}

template <int D>
__device__ __forceinline__ void load_state(const float* st, int stride, float& mx, float& z, float (&acc)[D / 4]) {
    mx = st[0];
    z = st[stride];
#pragma unroll
    for (int k = 0; k < D / 4; ++k) acc[k] = st[(2 + k) * stride];
}

template <int D>
__device__ __forceinline__ void store_state(float* st, int stride, float mx, float z, const float (&acc)[D / 4]) {
    st[0] = mx;
    st[stride] = z;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) st[(2 + k) * stride] = acc[k];
}

template <int D>
__device__ __forceinline__ void fold_into_smem(float* st, int stride, float lc, const float (&mc)[D / 4]) {
    float mx, z, acc[D / 4];
    load_state<D>(st, stride, mx, z, acc);
    fold_child<D>(mx, z, acc, lc, mc);
    store_state<D>(st, stride, mx, z, acc);
}

template <int D>
__device__ __forceinline__ void reset_smem(float* st, int stride) {
    st[0] = -INFINITY;
    st[stride] = 0.0f;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) st[(2 + k) * stride] = 0.0f;
}

// Key rows of a worker's span are staged in shared memory by cp.async, kStages groups of
// kTok tokens in flight, so the sequential per-token update reads K at shared-memory
// latency instead of waiting on global loads.
constexpr int kTok = 8;
constexpr int kStages = 3;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Streams the C^k_emit tokens of one level-k_emit node per worker and emits the summaries of
// every node of levels 1..k_emit beneath it.  Level-1 state lives in registers, levels
// 2..k_emit in shared memory ([level][field][thread]).
template <int D, int FMT>
__global__ void __launch_bounds__(128, 4) k_build_stream(BuildArgs a) {
    extern __shared__ float smem_state[];
    const int wt = 4 * a.R;
    const int wpb = blockDim.x / wt;
    const int tid = threadIdx.x;
    const int wk = tid / wt, wl = tid % wt;          // worker in block, thread in worker
    const int r = wl >> 2;
    const int q = tid & 3;
    int64_t widx = (int64_t)blockIdx.x * wpb + wk;
    const int64_t total = (int64_t)a.Hkv * a.nu;
    const bool active = widx < total;
    if (!active) widx = total - 1;
    const int g = (int)(widx / a.nu);
    const int64_t u = a.u0 + widx % a.nu;
    const int C = a.C;

    float qv[D / 4];
    load_row_bf16<D>(a.qref + ((int64_t)g * a.R + r) * D, q, qv);

    const int nst = a.k_emit - 1;   // shared-memory levels (2..k_emit)
    const int stride = blockDim.x;
    for (int l = 0; l < nst; ++l) reset_smem<D>(smem_state + (int64_t)l * (D / 4 + 2) * stride + tid, stride);
    // staged key rows: [worker][stage][token][D] bf16 after the level states
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_state + (int64_t)nst * (D / 4 + 2) * stride) +
                        (int64_t)wk * kStages * kTok * D;

    int64_t span_emit = 1;
    for (int l = 0; l < a.k_emit; ++l) span_emit *= C;
    const int64_t t0 = u * span_emit;
    const __nv_bfloat16* Kg = a.K + ((int64_t)g * a.ld + t0) * D;
    const int ngrp = (int)((span_emit + kTok - 1) / kTok);
    constexpr int kChunks = kTok * D * 2 / 16;       // 16-byte pieces of one token group
    auto issue = [&](int grp) {
        if (grp < ngrp) {
            __nv_bfloat16* dst = sK + (grp % kStages) * kTok * D;
            const __nv_bfloat16* src = Kg + (int64_t)grp * kTok * D;
            const int64_t rest = span_emit - (int64_t)grp * kTok;
            const int64_t ntk = rest < kTok ? rest : kTok;
            for (int c = wl; c < kChunks; c += wt)
                if (c / (D * 2 / 16) < ntk) cp_async16(dst + c * 8, src + c * 8);
        }
        cp_async_commit();   // one group per call on every thread keeps the counts aligned
    };
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) issue(i);

    float mx = -INFINITY, z = 0.0f, acc[D / 4];
#pragma unroll
    for (int k = 0; k < D / 4; ++k) acc[k] = 0.0f;

    int left = C;   // tokens left in the current level-1 chunk
    for (int grp = 0; grp < ngrp; ++grp) {
        issue(grp + kStages - 1);
        cp_async_wait<kStages - 1>();
        __syncthreads();
        const __nv_bfloat16* kb = sK + (grp % kStages) * kTok * D;
        const int64_t rest = span_emit - (int64_t)grp * kTok;
        const int ntk = (int)(rest < kTok ? rest : kTok);
        for (int tk = 0; tk < ntk; ++tk) {
            const int64_t tt = (int64_t)grp * kTok + tk;
            // packed fp32x2 arithmetic: two independent IEEE single-precision operations per
            // instruction (dims 2j, 2j+1 of this thread's D/4)
            float2 kv[D / 8];
            {
                const uint2* p = reinterpret_cast<const uint2*>(kb + tk * D);
#pragma unroll
                for (int i = 0; i < D / 16; ++i) {
                    const uint2 uu = p[4 * i + q];
                    kv[2 * i + 0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uu.x));
                    kv[2 * i + 1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uu.y));
                }
            }
            // q_r.k_t over this thread's dims as two interleaved partial sums
            float2 d2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < D / 8; ++j) d2 = __ffma2_rn(make_float2(qv[2 * j], qv[2 * j + 1]), kv[j], d2);
            const float sc = a.scale * quad_sum(d2.x + d2.y);
            const float mn = fmaxf(mx, sc);
            const float c = expf(mx - mn);
            const float wgt = expf(sc - mn);
            z = fmaf(z, c, wgt);
            {
                const float2 c2 = make_float2(c, c), w2 = make_float2(wgt, wgt);
#pragma unroll
                for (int j = 0; j < D / 8; ++j) {
                    const float2 a2 = __ffma2_rn(make_float2(acc[2 * j], acc[2 * j + 1]), c2, __fmul2_rn(w2, kv[j]));
                    acc[2 * j] = a2.x;
                    acc[2 * j + 1] = a2.y;
                }
            }
            mx = mn;
            if (--left == 0) {
                left = C;
                const int64_t t = t0 + tt;
                const int64_t j1 = t / C;
                float m1[D / 4];
                const float l1 = finalize_store<D>(mx, z, acc, qv, a.scale,
                                                   a.rec[1] + ((int64_t)g * a.cap[1] + j1) * a.ns,
                                                   a.lse[1] + ((int64_t)g * a.cap[1] + j1) * a.R, r, q, a.R,
                                                   active, a.rflag, m1, FMT);
                if (nst > 0) fold_into_smem<D>(smem_state + tid, stride, l1, m1);
                mx = -INFINITY;
                z = 0.0f;
#pragma unroll
                for (int k = 0; k < D / 4; ++k) acc[k] = 0.0f;
                // cascade completed ancestors (levels 2..k_emit)
                int64_t span = C;
                for (int l = 2; l <= a.k_emit; ++l) {
                    span *= C;
                    if ((tt + 1) % span != 0) break;
                    float* st = smem_state + (int64_t)(l - 2) * (D / 4 + 2) * stride + tid;
                    float smx, sz, sacc[D / 4], ml[D / 4];
                    load_state<D>(st, stride, smx, sz, sacc);
                    const int64_t jl = t / span;
                    const float ll = finalize_store<D>(smx, sz, sacc, qv, a.scale,
                                                       a.rec[l] + ((int64_t)g * a.cap[l] + jl) * a.ns,
                                                       a.lse[l] + ((int64_t)g * a.cap[l] + jl) * a.R, r, q, a.R,
                                                       active, a.rflag, ml, FMT);
                    if (l < a.k_emit)
                        fold_into_smem<D>(smem_state + (int64_t)(l - 1) * (D / 4 + 2) * stride + tid, stride, ll, ml);
                    reset_smem<D>(st, stride);
                }
            }
        }
        __syncthreads();   // stage grp % kStages is refilled by the next iteration's issue
    }
    cp_async_wait<0>();
}

// Merges the C children (level l-1) of each parent node P in [p0, p0+np) at level l:
// lse_P = log sum_c exp(lse_c), m_P = sum_c exp(lse_c - lse_P) m_c, b_P = lse_P - s q_r.m_P.
template <int D, int FMT>
__global__ void __launch_bounds__(128) k_merge(MergeArgs a) {
    const int wt = 4 * a.R;
    const int wpb = blockDim.x / wt;
    const int tid = threadIdx.x;
    const int r = (tid % wt) >> 2;
    const int q = tid & 3;
    int64_t widx = (int64_t)blockIdx.x * wpb + tid / wt;
    const int64_t total = (int64_t)a.Hkv * a.np;
    const bool active = widx < total;
    if (!active) widx = total - 1;
    const int g = (int)(widx / a.np);
    const int64_t P = a.p0 + widx % a.np;

    float qv[D / 4];
    load_row_bf16<D>(a.qref + ((int64_t)g * a.R + r) * D, q, qv);

    const float* crec = a.child_rec + ((int64_t)g * a.child_cap + P * a.C) * a.ns;
    const float* clse = a.child_lse + ((int64_t)g * a.child_cap + P * a.C) * a.R;
    float mx = -INFINITY, z = 0.0f, acc[D / 4], mc[D / 4], mo[D / 4];
#pragma unroll
    for (int k = 0; k < D / 4; ++k) acc[k] = 0.0f;
    for (int c = 0; c < a.C; ++c) {
        load_row_m<D>(crec + (int64_t)c * a.ns, a.R, r, q, mc, FMT);
        const float lc = __ldg(clse + (int64_t)c * a.R + r);
        fold_child<D>(mx, z, acc, lc, mc);
    }
    finalize_store<D>(mx, z, acc, qv, a.scale, a.rec + ((int64_t)g * a.cap + P) * a.ns,
                      a.lse + ((int64_t)g * a.cap + P) * a.R, r, q, a.R, active, a.rflag, mo, FMT);
}

// Decodes the m planes of nodes [0, n) of every KV head into f32 [Hkv][n][R][d].
__global__ void k_export_m(const float* rec, int64_t cap, int32_t ns, int32_t Hkv, int32_t R, int32_t d, int32_t fmt,
                           int64_t n, float* m) {
    const int64_t per = (int64_t)R * d / 4;   // float4 per node
    const int64_t total = (int64_t)Hkv * n * per;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t node = t / per, e4 = t % per;
        const int64_t h = node / n, j = node % n;
        const int r = (int)(e4 * 4 / d), k = (int)(e4 * 4 % d);
        const float4 v = m_load4(rec + (h * cap + j) * ns, R, d, r, k, fmt);
        reinterpret_cast<float4*>(m)[t] = v;
    }
}

int workers_per_block(int R) {
    const int wt = 4 * R;
    return wt >= 128 ? 1 : 128 / wt;
}

}  // namespace

cudaError_t launch_export_m(const float* rec, int64_t cap, int32_t ns, int32_t Hkv, int32_t R, int32_t d, int32_t fmt,
                            int64_t n, float* m, cudaStream_t st) {
    const int64_t total = (int64_t)Hkv * n * R * d / 4;
    if (total <= 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, sm_count() * 16);
    k_export_m<<<(unsigned)blocks, 256, 0, st>>>(rec, cap, ns, Hkv, R, d, fmt, n, m);
    return cudaGetLastError();
}

cudaError_t launch_build_stream(const BuildArgs& a, int d, cudaStream_t st) {
    if (a.nu <= 0) return cudaSuccess;
    const int wpb = workers_per_block(a.R);
    const int threads = wpb * 4 * a.R;
    const int64_t blocks = ((int64_t)a.Hkv * a.nu + wpb - 1) / wpb;
    const size_t smem = (size_t)(a.k_emit - 1) * (d / 4 + 2) * threads * sizeof(float) +
                        (size_t)wpb * kStages * kTok * d * 2;
    ProfScope ps_("k_build_stream", st);
    auto go = [&](auto kern) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<(unsigned)blocks, threads, smem, st>>>(a);
    };
    // one instance per head dimension and record format (the format's code only)
    if (d == 128) {
        if (a.fmt == kFmtBf16) go(k_build_stream<128, kFmtBf16>);
        else if (a.fmt == kFmtFp4) go(k_build_stream<128, kFmtFp4>);
        else go(k_build_stream<128, kFmtF16x2>);
    } else {
        if (a.fmt == kFmtBf16) go(k_build_stream<64, kFmtBf16>);
        else if (a.fmt == kFmtFp4) go(k_build_stream<64, kFmtFp4>);
        else go(k_build_stream<64, kFmtF16x2>);
    }
    return cudaGetLastError();
}

cudaError_t launch_merge(const MergeArgs& a, int d, cudaStream_t st) {
    if (a.np <= 0) return cudaSuccess;
    const int wpb = workers_per_block(a.R);
    const int threads = wpb * 4 * a.R;
    const int64_t blocks = ((int64_t)a.Hkv * a.np + wpb - 1) / wpb;
    ProfScope ps_("k_merge", st);
    auto go = [&](auto kern) { kern<<<(unsigned)blocks, threads, 0, st>>>(a); };
    if (d == 128) {
        if (a.fmt == kFmtBf16) go(k_merge<128, kFmtBf16>);
        else if (a.fmt == kFmtFp4) go(k_merge<128, kFmtFp4>);
        else go(k_merge<128, kFmtF16x2>);
    } else {
        if (a.fmt == kFmtBf16) go(k_merge<64, kFmtBf16>);
        else if (a.fmt == kFmtFp4) go(k_merge<64, kFmtFp4>);
        else go(k_merge<64, kFmtF16x2>);
    }
    return cudaGetLastError();
}

}  // namespace zha
