// zha_noalloc.cu - exact sparse attention over a routed token set without any device
// allocation: the working memory lives in one file-scope static device array.
//
// Who needs this: code that must not call cudaMalloc at the point where it attends -
// for example a host process that runs under a memory manager owning every device
// allocation, or a latency-critical loop where an allocation (and the implicit device
// synchronisation it can trigger) is not acceptable.  Such a caller passes its own
// inputs and outputs; the scratch below (group union lists, per-split partial softmax
// states, counters, the one-sequence table the kernels read) is reserved once when the
// library is loaded on a device and stays reserved until the process exits.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "zha_common.cuh"
#include "zha_launch.h"

namespace zha {

// Fixed working memory of zha_sparse_attn_static, shared by every call on a device.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

std::mutex g_static_mu;
void* g_static_ptr[64] = {nullptr};   // device address of g_static_scratch, per device ordinal
// Host side of each call, per device ordinal: the one-sequence table the kernels read (its
// upload reads this memory, which stays valid after the call returns) and the status word
// read back at the end of the call.
SeqDev g_static_seq[64];
int32_t g_static_status[64];

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

}  // namespace zha

using namespace zha;

static zha_status sfail(zha_status s, const char* msg) { return set_last_error(s, msg); }

extern "C" zha_status zha_sparse_attn_static(const void* K, const void* V, int64_t ld, int64_t n_tokens,
                                             int32_t C, int32_t L, int32_t Hq, int32_t Hkv, int32_t d,
                                             const void* Q, int32_t n_q, const uint32_t* kept1, int64_t words,
                                             float* out, void* stream) {
    auto aligned16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!K || !V || !Q || !kept1 || !out) return sfail(ZHA_ERR_ARG, "K, V, Q, kept1 and out must be non-NULL");
    if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(out) || !aligned16(kept1))
        return sfail(ZHA_ERR_ARG, "device pointers must be 16-byte aligned");
    if (C < 2 || C > 1024 || L < 1 || L > kMaxL) return sfail(ZHA_ERR_ARG, "C must be in [2, 1024], L in [1, 16]");
    if (d != 64 && d != 128) return sfail(ZHA_ERR_ARG, "d must be 64 or 128");
    if (Hkv < 1 || Hq < Hkv || Hq % Hkv) return sfail(ZHA_ERR_ARG, "Hq must be a positive multiple of Hkv");
    if (n_q < 1) return sfail(ZHA_ERR_ARG, "n_q must be >= 1");
    if (n_tokens < 1 || n_tokens > ld) return sfail(ZHA_ERR_ARG, "need 1 <= n_tokens <= ld");
    int64_t top = 1;
    for (int l = 0; l < L; ++l) top = top > (int64_t(1) << 40) / C ? (int64_t(1) << 41) : top * C;
    const int64_t n1 = n_tokens / C;
    if (words < (n1 + 31) / 32) return sfail(ZHA_ERR_ARG, "words must cover n_tokens / C bits");

    // Working memory needed by this call, carved from the static array.
    const int64_t lanes = (int64_t)n_q * Hq;
    const int n_gl = n_q * (Hq / Hkv);
    const int64_t nseg = 1 + n1 + (std::min<int64_t>(top, n_tokens) + C - 1) / C;
    const int64_t segs = segs_per_split(n_gl, C);
    const int64_t splits = (nseg + segs - 1) / segs;
    size_t off = 0;
    const size_t seq_off = off;     off += up256(sizeof(SeqDev));
    const size_t ctr_off = off;     off += up256((size_t)kCtrCount * 8);
    const size_t status_off = off;  off += up256(4);
    const size_t ucount_off = off;  off += up256((size_t)Hkv * 4);
    const size_t ulist_off = off;   off += up256((size_t)Hkv * std::max<int64_t>(n1, 1) * 4);
    const int64_t uw = std::max<int64_t>(words, 1);
    const size_t uword_off = off;   off += up256((size_t)Hkv * uw * 4);
    const size_t kcount_off = off;  off += up256((size_t)(kMaxL + 1) * lanes * 4);
    const size_t part_off = off;    off += up256((size_t)lanes * splits * (d + 4) * 4);
    if (off > kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "call needs %zu bytes of working memory, the static array holds %zu "
                 "(fewer query tokens or a shorter cache per call)", off, kStaticScratchBytes);
        return sfail(ZHA_ERR_CAPACITY, msg);
    }

    // Device address of the static array for the current device (looked up once per device).
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sfail(ZHA_ERR_CUDA, "cudaGetDevice failed");
    unsigned char* base = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_static_mu);
        if (!g_static_ptr[dev]) {
            void* p = nullptr;
            cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
            if (e != cudaSuccess || !p) return sfail(ZHA_ERR_CUDA, "cudaGetSymbolAddress(static scratch) failed");
            g_static_ptr[dev] = p;
        }
        base = static_cast<unsigned char*>(g_static_ptr[dev]);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    SeqDev& sd = g_static_seq[dev];
    memset(&sd, 0, sizeof(sd));
    sd.C = C;
    sd.L = L;
    sd.N = n_tokens;
    sd.top = top;
    sd.T = n_tokens / top;
    sd.ld = ld;
    int64_t span = 1;
    for (int l = 1; l <= L; ++l) {
        span = span > (int64_t(1) << 40) / C ? (int64_t(1) << 41) : span * C;
        sd.n[l] = n_tokens / span;
    }
    sd.K = static_cast<const __nv_bfloat16*>(K);
    sd.V = static_cast<const __nv_bfloat16*>(V);
    if (cudaMemcpyAsync(base + seq_off, &sd, sizeof(sd), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return sfail(ZHA_ERR_CUDA, "cudaMemcpyAsync(sequence table) failed");
    // Counters and the per-lane kept counts accumulate or are read as zero: clear them.
    if (cudaMemsetAsync(base + ctr_off, 0, part_off - ctr_off, st) != cudaSuccess)
        return sfail(ZHA_ERR_CUDA, "cudaMemsetAsync(static scratch) failed");

    Work w;
    memset(&w, 0, sizeof(w));
    w.kept[1] = const_cast<uint32_t*>(kept1);
    w.W[1] = words;
    w.kcount = reinterpret_cast<int32_t*>(base + kcount_off);
    w.lanes_cap = lanes;
    w.ulist = reinterpret_cast<int32_t*>(base + ulist_off);
    w.us = std::max<int64_t>(n1, 1);
    w.ucount = reinterpret_cast<int32_t*>(base + ucount_off);
    w.uword = reinterpret_cast<uint32_t*>(base + uword_off);
    w.uw = uw;
    w.part = reinterpret_cast<float*>(base + part_off);
    w.s_cap = splits;
    w.ctr = reinterpret_cast<unsigned long long*>(base + ctr_off);
    w.status = reinterpret_cast<int32_t*>(base + status_off);

    Batch b;
    memset(&b, 0, sizeof(b));
    b.seqs = reinterpret_cast<const SeqDev*>(base + seq_off);
    b.n_seq = 1;
    b.n_q = n_q;
    b.Hq = Hq;
    b.Hkv = Hkv;
    b.G = Hq / Hkv;
    b.d = d;
    b.n_gl = n_gl;
    b.n_lanes = (int32_t)lanes;
    b.n_groups = Hkv;
    b.Q = static_cast<const __nv_bfloat16*>(Q);
    b.p = 1.0f;
    b.attn_path = 1;   // CUDA-core attention: it reads the kept bitmaps directly, no lane masks

    const float scale = (float)(1.0 / sqrt((double)d));
    if (launch_union(b, w, 0, 1, st) != cudaSuccess || launch_attn(b, w, splits, scale, st) != cudaSuccess ||
        launch_combine(b, w, out, st) != cudaSuccess)
        return sfail(ZHA_ERR_CUDA, "kernel launch failed");
    // The call waits for its kernels and reads the device status word back (no kernel of this
    // path is expected to set it: the union keeps only chunks under complete top nodes).
    int32_t& hs = g_static_status[dev];
    hs = 0;
    if (cudaMemcpyAsync(&hs, base + status_off, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return sfail(ZHA_ERR_CUDA, "reading the device status word failed");
    if (hs) {
        char msg[96];
        snprintf(msg, sizeof(msg), "device status 0x%x (a union list reached its capacity)", (unsigned)hs);
        return sfail(ZHA_ERR_DEVICE, msg);
    }
    return ZHA_OK;
}
