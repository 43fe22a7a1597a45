// zha_common.cuh - device-side tables and helpers shared by the libzha kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zha.h"

namespace zha {

constexpr int kMaxL = ZHA_MAX_LEVELS;

// Node record layout in HBM (per level, per KV head, per node): the R slopes m_r in the tree's
// summary format, then b [R] f32; stride `ns` floats rounded up to 8 floats (32-byte
// sectors).  lse [R] f32 is kept in a separate array per level (read by merges and export).
//   format 0 (ZHA_SUMMARY_F16X2): m as fp16 planes hi [R][d] then lo [R][d] (4 bytes a value)
//   format 1 (ZHA_SUMMARY_BF16):  m as one bf16 plane [R][d] (2 bytes a value)
//   format 2 (ZHA_SUMMARY_FP4):   m as MXFP4 (the OCP microscaling format): E2M1 codes [R][d]
//                                 packed two to a byte (even dim in the low nibble), then one
//                                 E8M0 scale byte per block of 32 dims [R][d/32], that area
//                                 padded to 16 bytes (half a byte and 1/32 byte a value)
constexpr int kFmtF16x2 = 0;
constexpr int kFmtBf16 = 1;
constexpr int kFmtFp4 = 2;
constexpr int kFp4Block = 32;        // dims sharing one scale
// Floats of an MXFP4 record's scale area.
inline __host__ __device__ int64_t fp4_scale_floats(int R, int d) { return ((int64_t)R * d / kFp4Block + 15) / 16 * 4; }
inline __host__ __device__ int32_t record_stride(int R, int d, int fmt = kFmtF16x2) {
    if (fmt == kFmtFp4) return (int32_t)(((int64_t)R * d / 8 + fp4_scale_floats(R, d) + R + 7) / 8 * 8);
    return fmt == kFmtBf16 ? ((R * d / 2 + R + 7) / 8) * 8 : ((R * (d + 1) + 7) / 8) * 8;
}
// Floats from the start of a record to its b values.
inline __host__ __device__ int64_t b_offset(int R, int d, int fmt) {
    if (fmt == kFmtFp4) return (int64_t)R * d / 8 + fp4_scale_floats(R, d);
    return fmt == kFmtBf16 ? (int64_t)R * d / 2 : (int64_t)R * d;
}
// Bytes a scorer reads per node: the m planes (codes and scales) and b.
inline __host__ __device__ int64_t scored_node_bytes(int R, int d, int fmt) {
    if (fmt == kFmtFp4) return (int64_t)R * d / 2 + (int64_t)R * d / kFp4Block + (int64_t)R * 4;
    return (fmt == kFmtBf16 ? (int64_t)R * d * 2 : (int64_t)R * d * 4) + (int64_t)R * 4;
}

// One sequence of a decode batch, as the kernels see it.
struct SeqDev {
    int32_t C, L, R, ns;
    int32_t fmt;                     // summary format of the tree (kFmtF16x2 / kFmtBf16)
    int64_t N;                       // tokens present
    int64_t T;                       // complete top-level nodes = N / C^L
    int64_t top;                     // C^L
    int64_t ld;                      // K/V rows per KV head (capacity)
    int64_t n[kMaxL + 1];            // complete nodes per level (index = level)
    int64_t cap[kMaxL + 1];          // node capacity per level
    const float* rec[kMaxL + 1];     // [Hkv][cap_l][ns] node records (layout below)
    const int32_t* rflag;            // tree's range flag: a summary left the fp16 range
    const __nv_bfloat16* K;          // [Hkv][ld][d]
    const __nv_bfloat16* V;
    int32_t no_sink;                 // 1: token 0 of this tree is not the sequence's first token
                                     // (a later shard of a sharded sequence): no sink segment
};

// Whether attention over the tree has the sink segment (token 0, attended every time): the
// tree holds a complete top node and starts the sequence.
__host__ __device__ inline int seq_has_sink(const SeqDev& sq) { return (sq.T >= 1 && !sq.no_sink) ? 1 : 0; }

constexpr int kMapsPerLevel = 3;     // planes by 1 node, planes by 4 nodes, b by 4 nodes

// Counter slots (unsigned long long).
constexpr int kCtrUnionNodes = 0;              // + level
constexpr int kCtrLaneNodes = kMaxL + 1;       // + level
constexpr int kCtrUnionTokens = 2 * kMaxL + 2;
constexpr int kCtrLaneTokens = 2 * kMaxL + 3;
constexpr int kCtrCount = 2 * kMaxL + 4;

// Decoder workspace as the kernels see it.
struct Work {
    uint32_t* kept[kMaxL + 2];       // kept[l]: [lanes_cap][W[l]] bitmaps
    int64_t W[kMaxL + 2];
    int32_t* kcount;                 // [(kMaxL+1)][lanes_cap]
    int64_t lanes_cap;
    float* e;                        // [lanes_cap][es] scores of the current level
    int64_t es;
    int32_t* ulist;                  // [groups_cap][us] union lists
    int64_t us;
    int32_t* ucount;                 // [groups_cap]
    uint32_t* uword;                 // [groups_cap][uw] union bitmap being built
    int64_t uw;
    float* part;                     // [lanes_cap][s_cap][d+2] attention partials
    int64_t s_cap;
    uint32_t* memb;                  // [groups_cap][ms][mwords] union parents' lane masks (tensor scorer)
    int64_t ms;
    int32_t mwords;                  // a multiple of 8 covering every 256-lane pair of a group
    const CUtensorMap* tmaps;        // [n_seq][kMaxL + 1][kMapsPerLevel] TMA maps of the trees' levels (or null)
    uint32_t* lane_max;              // [(kMaxL+1)][lanes_cap] frontier max score per lane (ordered bits)
    int32_t* lane_cnt;               // [(kMaxL+1)][lanes_cap] frontier size per lane
    unsigned long long* ctr;         // kCtrCount counters
    int32_t* status;                 // device status word (0 = ok)
    // Sequence-sharded routing (one sequence whose tokens are split over ranks; null / 0 on
    // every other path).  k_select then runs in one of three phases around the collectives:
    // 1 writes the lane's mass histogram, 2 cuts on the summed histogram and writes the
    // boundary bin's keys, 3 finishes the cut on every rank's keys.
    int32_t sh_phase;                // 0: the whole cut in one kernel
    int32_t sh_world;                // ranks
    int64_t sh_off;                  // global index of this rank's first node of the level
    unsigned long long* sh_hist;     // [lanes][kShardBins] fixed-point bin masses
    unsigned long long* sh_keys;     // [lanes][kShardKeys] boundary-bin keys (global node ids)
    int32_t* sh_nkeys;               // [lanes]
    const unsigned long long* sh_keys_all;   // [world][lanes][kShardKeys]
    const int32_t* sh_nkeys_all;     // [world][lanes]
    unsigned long long* sh_need;     // [lanes_cap] mass still needed from the boundary bin
    float* lse_out;                  // [lanes] log-sum-exp of each lane's attention (or null)
};

constexpr int kShardBins = 2048;     // histogram bins of the sharded cut (those of k_select)
constexpr int kShardKeys = 2048;     // boundary-bin keys one rank contributes per lane
constexpr int kShardMergeKeys = 4096;   // keys of all ranks one lane's finish can sort

// A decode call's shape.
struct Batch {
    const SeqDev* seqs;
    int32_t n_seq, n_q, Hq, Hkv, G, d;
    int32_t n_gl;                    // lanes per (sequence, KV head) group = n_q * G
    int32_t n_lanes, n_groups;
    const __nv_bfloat16* Q;          // [n_seq][n_q][Hq][d]
    float p;
    int32_t score_path;              // 0 auto, 1 CUDA cores, 2 tensor cores (R = 16 only)
    int32_t attn_path;               // 0 auto, 1 CUDA cores, 2 tensor cores
    int32_t all_r16;                 // every tree of the batch has R = 16
    int32_t fmt = 0;                 // summary format shared by the batch's trees
    int32_t dense = 0;               // every lane attends every token (no routed sets, no lane masks)
    int32_t split_tok = 0;           // attention split size in tokens (0: split_tokens(n_gl))
};

// Global lane index of group lane y of group (s, g): lane = (s*n_q + i)*Hq + h.
__host__ __device__ inline int64_t lane_of(const Batch& b, int s, int g, int y) {
    const int i = y / b.G, hh = y % b.G;
    return ((int64_t)s * b.n_q + i) * b.Hq + (int64_t)g * b.G + hh;
}

// Node record (ns floats): the R reference-query means m_r are stored as two fp16 planes,
// hi [R][d] = fp16(m) then lo [R][d] = fp16(m - hi), followed by b [R] (f32).  hi + lo
// recovers m within 2^-22 |m| + 2^-25 (exactly representable in f32), and the planes are
// the tensor cores' operand format.  |m| must stay below 65504.
__device__ __forceinline__ void m_encode2(float a, float b, uint32_t& hi, uint32_t& lo, float& da, float& db) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
    const float2 lf = __half22float2(l);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
    da = hf.x + lf.x;
    db = hf.y + lf.y;
}
__device__ __forceinline__ float2 m_decode2(uint32_t hi, uint32_t lo) {
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    const float2 lf = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    return make_float2(hf.x + lf.x, hf.y + lf.y);
}
// The same for a one-plane bf16 record: two bf16 values of a 32-bit word.
__device__ __forceinline__ float2 m_decode_bf16(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}
// MXFP4 (OCP Microscaling Formats specification v1.0, the MXFP4 element and scale types and
// the conversion to them): a block of 32 values shares the scale X = 2^(floor(log2 amax) - 2)
// (2 = the largest exponent of E2M1), stored as its E8M0 byte floor(log2 amax) - 2 + 127
// (clamped at 0: a zero or tiny block); each value is v / X rounded to the nearest E2M1 value
// {0, 0.5, 1, 1.5, 2, 3, 4, 6} (ties to the even code, magnitudes above 6 saturate to 6) with
// v's sign (no negative zero).
__host__ __device__ inline uint32_t fp4_scale_byte(float amax) {
    union { float f; uint32_t u; } c;
    c.f = amax;
    const int ex = (int)((c.u >> 23) & 0xFFu);      // floor(log2 amax) + 127 for a normal amax
    return (uint32_t)(ex >= 2 ? (ex > 255 ? 253 : ex - 2) : 0);
}
// 2^(E - 127) and 2^(127 - E) for an E8M0 byte E in [0, 253].
__host__ __device__ inline float fp4_scale(uint32_t E) {
    union { float f; uint32_t u; } c;
    c.u = E ? (E << 23) : 0x00400000u;             // E = 0: 2^-127, a subnormal float
    return c.f;
}
__host__ __device__ inline float fp4_inv_scale(uint32_t E) {
    union { float f; uint32_t u; } c;
    c.u = (254u - E) << 23;
    return c.f;
}
// E2M1 code of y (already divided by the scale): the count of rounding boundaries below |y|,
// a tie counting when the upper neighbour has the even code.
__host__ __device__ inline uint32_t fp4_code(float y) {
    const float a = fabsf(y);
    const uint32_t c = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                       (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.0f);
    return c | ((c != 0u && y < 0.0f) ? 8u : 0u);
}
// Value of an E2M1 code (bit 3 sign, bits 2-1 exponent, bit 0 mantissa) times a scale.
__host__ __device__ inline float fp4_value(uint32_t code, float scale) {
    const uint32_t e = (code >> 1) & 3u, m = code & 1u;
    uint32_t bits = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
    bits |= (code & 8u) << 28;
    union { float f; uint32_t u; } c;
    c.u = bits;
    return c.f * scale;
}
// Byte pointers of an MXFP4 record: the codes and the scales.
__device__ __forceinline__ const uint8_t* fp4_codes(const float* rec) { return reinterpret_cast<const uint8_t*>(rec); }
__device__ __forceinline__ const uint8_t* fp4_scales(const float* rec, int R, int D) {
    return reinterpret_cast<const uint8_t*>(rec) + (int64_t)R * D / 2;
}
// Four consecutive values (dims k..k+3, k a multiple of 4) of slope r of an MXFP4 record.
__device__ __forceinline__ float4 fp4_load4(const float* rec, int R, int D, int r, int k) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(fp4_codes(rec) + ((int64_t)r * D + k) / 2);
    const float X = fp4_scale(fp4_scales(rec, R, D)[(int64_t)r * (D / kFp4Block) + k / kFp4Block]);
    return make_float4(fp4_value(w & 15u, X), fp4_value((w >> 4) & 15u, X), fp4_value((w >> 8) & 15u, X),
                       fp4_value((w >> 12) & 15u, X));
}

// Four consecutive m values (dims k..k+3 of slope r) of a record in format fmt.
__device__ __forceinline__ float4 m_load4(const float* rec, int R, int D, int r, int k, int fmt) {
    if (fmt == kFmtFp4) return fp4_load4(rec, R, D, r, k);
    if (fmt == kFmtBf16) {
        const uint2 a = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(rec) + (int64_t)r * D + k);
        const float2 x = m_decode_bf16(a.x), y = m_decode_bf16(a.y);
        return make_float4(x.x, x.y, y.x, y.y);
    }
    const __half* h = reinterpret_cast<const __half*>(rec);
    const uint2 a = *reinterpret_cast<const uint2*>(h + (int64_t)r * D + k);
    const uint2 c = *reinterpret_cast<const uint2*>(h + (int64_t)R * D + (int64_t)r * D + k);
    const float2 x = m_decode2(a.x, c.x), y = m_decode2(a.y, c.y);
    return make_float4(x.x, x.y, y.x, y.y);
}

// Order-preserving map of a float to uint32 (atomicMax on the result is a float max).
__host__ __device__ inline uint32_t ord_bits(float f) {
    union { float f; uint32_t u; } c;
    c.f = f;
    return (c.u & 0x80000000u) ? ~c.u : (c.u | 0x80000000u);
}
__host__ __device__ inline float unord_bits(uint32_t o) {
    union { float f; uint32_t u; } c;
    c.u = (o & 0x80000000u) ? (o ^ 0x80000000u) : ~o;
    return c.f;
}

// Device status bits.
constexpr int32_t kStatusSelectFallbackLimit = 1;
constexpr int32_t kStatusCapacity = 2;
constexpr int32_t kStatusTimeout = 4;        // a bounded wait on the tensor-core pipeline gave up
constexpr int32_t kStatusRange = 8;          // an entry of Q or of a summary exceeds the fp16 range
constexpr int32_t kStatusShardKeys = 16;     // a sharded cut's boundary bin held more keys than it can exchange

// Streaming multiprocessors of the current device (grids are sized in multiples of it);
// looked up once per device ordinal.
inline int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// A tree's flag word as routing reports it: bit 0, a summary left the fp16 range (kStatusRange);
// bit 1, a wait of the tensor-core build gave up (kStatusTimeout: the tree is incomplete).
__device__ __forceinline__ void tree_flag_status(int32_t flag, int32_t* status) {
    if (flag) atomicOr(status, ((flag & 1) ? kStatusRange : 0) | ((flag & 2) ? kStatusTimeout : 0));
}

// Split size (tokens) of the attention work for a call with n_gl lanes per group.
inline __host__ __device__ int split_tokens(int n_gl) { return n_gl <= 64 ? 1024 : 4096; }
inline __host__ __device__ int64_t segs_per_split(int n_gl, int C) {
    const int64_t s = split_tokens(n_gl) / C;
    return s > 0 ? s : 1;
}
// Split size of a decoder call: on the CUDA-core attention, groups of a few lanes take short
// splits (more warps in flight over a small kept set); the tensor-core attention keeps
// split_tokens (its CTAs gather 128-position tiles, so longer splits amortise each CTA's
// set-up).  The partials workspace is sized by lanes x splits.
inline __host__ __device__ int decoder_split_tokens(int n_gl) { return n_gl <= 16 ? 256 : split_tokens(n_gl); }
inline __host__ __device__ int64_t batch_segs(const Batch& b, int C) {
    const int64_t s = (b.split_tok > 0 ? b.split_tok : split_tokens(b.n_gl)) / C;
    return s > 0 ? s : 1;
}

}  // namespace zha
