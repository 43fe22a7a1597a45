// zha_launch.h - kernel argument blocks and launchers (internal to libzha).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zha_common.cuh"

namespace zha {

// Streaming build: workers summarise level-k_emit nodes [u0, u0+nu) of every KV head and
// write levels 1..k_emit beneath them.
struct BuildArgs {
    const __nv_bfloat16* K;      // [Hkv][ld][d]
    int64_t ld;
    const __nv_bfloat16* qref;   // [Hkv][R][d]
    int32_t* rflag;              // set when a summary leaves the fp16 range
    int32_t Hkv, R, C, ns, k_emit;
    int32_t fmt;                 // summary format (kFmtF16x2 / kFmtBf16)
    int64_t u0, nu;
    float scale;
    float* rec[kMaxL + 1];
    float* lse[kMaxL + 1];
    int64_t cap[kMaxL + 1];
};

// Merge: parents [p0, p0+np) of one level from their C children.
struct MergeArgs {
    const __nv_bfloat16* qref;
    int32_t* rflag;
    int32_t Hkv, R, C, ns;
    int32_t fmt;
    int64_t p0, np;
    float scale;
    const float* child_rec;
    const float* child_lse;
    int64_t child_cap;
    float* rec;
    float* lse;
    int64_t cap;
};

// Tensor-core build (C = 4, R = 16, d = 64 or 128): tiles [t0, t1) of 128 tokens of every KV
// head; writes every complete node of levels 1..k_emit (k_emit <= 3) whose tokens lie in them.
struct BuildTcArgs {
    const __nv_bfloat16* K;      // [Hkv][ld][d]
    int64_t ld, n_tokens;        // rows of the cache valid for this call
    const __nv_bfloat16* qref;   // [Hkv][R][d]
    int32_t* rflag;              // bit 0: a summary left the fp16 range; bit 1: a wait gave up
    int32_t Hkv, ns, k_emit;
    int64_t t0, t1;
    int64_t n1, n2, n3;          // complete nodes of levels 1..3 (n_tokens / C^l)
    float scale;
    float* rec[4];
    float* lse[4];
    int64_t cap[4];
};

cudaError_t launch_build_stream(const BuildArgs& a, int d, cudaStream_t st);
bool build_tc_supported(int C, int R, int d, int fmt);
cudaError_t launch_build_tc(const BuildTcArgs& a, int d, cudaStream_t st);
cudaError_t launch_merge(const MergeArgs& a, int d, cudaStream_t st);
// m of nodes [0, n) of every KV head of one level, decoded to f32 [Hkv][n][R][d].
cudaError_t launch_export_m(const float* rec, int64_t cap, int32_t ns, int32_t Hkv, int32_t R, int32_t d, int32_t fmt,
                            int64_t n, float* m, cudaStream_t st);

// Decode (routing + attention).  `it` is the level iteration: sequence s works on level
// L_s - it.  mode 0 of the union kernel prepares routing iteration it (union of the kept
// sets of level L_s - it + 1); mode 1 prepares attention (union of level-1 kept sets).
cudaError_t launch_union(const Batch& b, const Work& w, int it, int mode, cudaStream_t st);
cudaError_t launch_score(const Batch& b, const Work& w, int it, float scale, cudaStream_t st);
// Transposed lane masks of a union level (mode 0: parents of iteration it's candidates;
// mode 1: kept level-1 chunks) into w.memb.
cudaError_t launch_member(const Batch& b, const Work& w, int it, int mode, cudaStream_t st);
cudaError_t launch_score_tc(const Batch& b, const Work& w, int it, float scale, cudaStream_t st);
// Lanes per group from which the automatic choice scores on tensor cores.
// max_cands: an upper bound on any lane's candidates at this iteration (picks the block size).
cudaError_t launch_select(const Batch& b, const Work& w, int it, int64_t max_cands, cudaStream_t st);
cudaError_t launch_attn(const Batch& b, const Work& w, int64_t max_splits, float scale, cudaStream_t st);
cudaError_t launch_attn_tc(const Batch& b, const Work& w, int64_t max_splits, float scale, cudaStream_t st);
// Whether a call's attention runs on the tensor cores: forced, or the automatic choice, which
// takes them at every lane count (a padded 128-lane tile measured faster than the CUDA-core
// split-KV kernel even for one query token).  Calls with more than 65,535 splits use the
// CUDA-core kernel either way.
inline bool attn_on_tensor_cores(const Batch& b) { return b.attn_path == 2 || b.attn_path == 0; }
cudaError_t launch_combine(const Batch& b, const Work& w, float* out, cudaStream_t st);

// Sharded sequence: a level's frontier maximum and size between the decoder's arrays and the
// exchange (to_exchange: ordered bits -> ordered int32; else back), and the ranks' merge of
// their attention outputs by log-sum-exp.
cudaError_t launch_shard_lanes(uint32_t* lane_max, int32_t* lane_cnt, int32_t* ex_max, int32_t* ex_cnt,
                               int64_t lanes, bool to_exchange, cudaStream_t st);
cudaError_t launch_shard_combine(const float* out_all, const float* lse_all, int64_t lanes, int world, int d,
                                 float* out, cudaStream_t st);

// Records the message returned by zha_last_error() on this thread; returns s.
zha_status set_last_error(zha_status s, const char* msg);

}  // namespace zha
