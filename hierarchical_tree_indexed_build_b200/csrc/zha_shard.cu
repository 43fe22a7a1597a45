// zha_shard.cu - the small kernels of a sequence whose tokens are split over ranks.
//
// Routing a sharded sequence takes each level's top-p cut over the union of every rank's
// frontier (fluxbbs.com "Zyphra ZHA 稀疏注意力…", section 树形索引是怎么搭的: keep the fewest
// nodes of the frontier whose mass reaches p); the per-level exchange is done by the caller's
// collectives between the select kernel's phases (zha_route.cu, k_select).  This file holds
// what surrounds them: the frontier maximum and size in and out of the exchange, and the
// final merge of the ranks' attention outputs.
#include <math.h>

#include "zha_common.cuh"
#include "zha_launch.h"
#include "zha_profile.h"

namespace zha {

namespace {

// Ordered float bits (unsigned order) <-> int32 whose signed order is the same: flip bit 31.
__global__ void k_shard_lanes(uint32_t* lane_max, int32_t* lane_cnt, int32_t* ex_max, int32_t* ex_cnt,
                              int64_t lanes, int to_exchange) {
    const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= lanes) return;
    if (to_exchange) {
        ex_max[x] = (int32_t)(lane_max[x] ^ 0x80000000u);
        ex_cnt[x] = lane_cnt[x];
    } else {
        lane_max[x] = (uint32_t)ex_max[x] ^ 0x80000000u;
        lane_cnt[x] = ex_cnt[x];
    }
}

// out[x] = sum_r exp(lse_r - M) out_r / sum_r exp(lse_r - M), M = max_r lse_r: the softmax over
// the union of the ranks' attended tokens, from each rank's normalised output and its
// log-sum-exp.  Ranks with no token for the lane (lse = -inf) are skipped.  One block of d
// threads per lane, ranks added in rank order.
__global__ void k_shard_combine(const float* __restrict__ out_all, const float* __restrict__ lse_all, int64_t lanes,
                                int world, int d, float* __restrict__ out) {
    const int64_t x = blockIdx.x;
    const int t = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < world; ++r) M = fmaxf(M, lse_all[(int64_t)r * lanes + x]);
    float num = 0.0f, den = 0.0f;
    if (M > -INFINITY) {
        for (int r = 0; r < world; ++r) {
            const float l = lse_all[(int64_t)r * lanes + x];
            if (l > -INFINITY) {
                const float c = expf(l - M);
                num = fmaf(c, out_all[((int64_t)r * lanes + x) * d + t], num);
                den += c;
            }
        }
    }
    out[x * d + t] = den > 0.0f ? num / den : 0.0f;
}

}  // namespace

cudaError_t launch_shard_lanes(uint32_t* lane_max, int32_t* lane_cnt, int32_t* ex_max, int32_t* ex_cnt,
                               int64_t lanes, bool to_exchange, cudaStream_t st) {
    if (lanes <= 0) return cudaSuccess;
    ProfScope ps_("k_shard_lanes", st);
    k_shard_lanes<<<(unsigned)((lanes + 255) / 256), 256, 0, st>>>(lane_max, lane_cnt, ex_max, ex_cnt, lanes,
                                                                  to_exchange ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_shard_combine(const float* out_all, const float* lse_all, int64_t lanes, int world, int d,
                                 float* out, cudaStream_t st) {
    if (lanes <= 0) return cudaSuccess;
    ProfScope ps_("k_shard_combine", st);
    k_shard_combine<<<(unsigned)lanes, d, 0, st>>>(out_all, lse_all, lanes, world, d, out);
    return cudaGetLastError();
}

}  // namespace zha
