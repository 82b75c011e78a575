// Internal launchers shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <tuple>

namespace lsa {

// Host-side caches so that a launch costs no driver attribute queries after
// the first call (per kernel, device and configuration).
inline int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
}

inline cudaError_t ensure_dyn_smem(const void* kern, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> done;
    const int dev = current_device();
    std::lock_guard<std::mutex> g(mu);
    int& cur = done[{kern, dev}];
    if (cur >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}

inline cudaError_t cached_occupancy(const void* kern, int threads, size_t smem, int* occ) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> done;
    const int dev = current_device();
    std::lock_guard<std::mutex> g(mu);
    auto key = std::make_tuple(kern, dev, threads, smem);
    auto it = done.find(key);
    if (it != done.end()) {
        *occ = it->second;
        return cudaSuccess;
    }
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kern, threads, smem);
    if (e == cudaSuccess) done[key] = *occ;
    return e;
}

// Clusters of cfg's shape that can be resident at once (cached per kernel,
// device and configuration).
inline cudaError_t cached_active_clusters(const void* kern, const cudaLaunchConfig_t& cfg, int* clusters) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, unsigned, unsigned, size_t>, int> done;
    const int dev = current_device();
    unsigned cx = 1;
    for (unsigned i = 0; i < cfg.numAttrs; ++i)
        if (cfg.attrs[i].id == cudaLaunchAttributeClusterDimension) cx = cfg.attrs[i].val.clusterDim.x;
    std::lock_guard<std::mutex> g(mu);
    auto key = std::make_tuple(kern, dev, cfg.blockDim.x, cx, cfg.dynamicSmemBytes);
    auto it = done.find(key);
    if (it != done.end()) {
        *clusters = it->second;
        return cudaSuccess;
    }
    cudaError_t e = cudaOccupancyMaxActiveClusters(clusters, kern, &cfg);
    if (e == cudaSuccess) done[key] = *clusters;
    return e;
}

// 2-D bf16 tensor map over `outer` rows of `inner` elements, rows `row_bytes`
// apart, boxes of box_inner x box_outer, swizzled to the box row width (32,
// 64 or 128 bytes). Returns false if the driver entry point or the encoding
// fails.
bool make_tensor_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                        uint32_t box_inner, uint32_t box_outer);

struct LaunchCtx {
    cudaStream_t stream;
    int num_sms;
    long long wait_limit;
};

struct AttnPlan {
    long long units;          // rows x KV heads
    int tiles_per_unit;       // ceil(B / 64)
    long long total_tiles;
    int ctas;                 // persistent CTAs (one wave)
    int smax;                 // partial slots per unit
};

// mode 0: scores are the group-sum dot products (G x the mean); mode 1: means.
// ghist (optional, [batch * hkv, 2048], zero on entry): the scorer may add the
// histogram of the top 11 order-key bits of the scores it writes; *hist_done
// tells whether it did (only some shapes support it).
cudaError_t launch_score(const LaunchCtx& ctx, const uint16_t* qt, const uint16_t* kt, float* out, int batch, int hq,
                         int hkv, int r, int n, int mode, unsigned* status, uint32_t* ghist = nullptr,
                         bool* hist_done = nullptr);

// As launch_score with kt stored as OCP FP8 E4M3 (1 byte per value); r must be
// 64 and hkv one of 4, 8, 16, 32 (else cudaErrorInvalidValue, nothing launched).
cudaError_t launch_score_fp8(const LaunchCtx& ctx, const uint16_t* qt, const uint8_t* kt, float* out, int batch,
                             int hq, int hkv, int r, int n, int mode, unsigned* status, uint32_t* ghist = nullptr,
                             bool* hist_done = nullptr);

cudaError_t launch_fine_score(const LaunchCtx& ctx, const uint16_t* qt, const uint16_t* kt, const int32_t* blk_idx,
                              int keep, int blk, float* out, int batch, int hq, int hkv, int r, int T);

cudaError_t launch_centroids(const LaunchCtx& ctx, const uint16_t* kt, int blk, uint16_t* cen, int batch, int hkv, int r,
                             int T);

// ghist (optional): the rows' histograms of key >> 21 from launch_score; the
// kernel zeroes them after use.
cudaError_t launch_topk(const LaunchCtx& ctx, const float* scores, int rows, int n, int B, int32_t* idx,
                        const int32_t* blkmap, int blk, int keep, uint32_t* ghist = nullptr);

// Scoring preparation (project.cu). y[b, t, i, :] = P[i / (H / nbases)] x[b, t, i, :]
// for t in [t0, t0 + n) of every sequence: x [batch, T, H, d] bf16, P
// [nbases, r, d] bf16, y [batch, T, H, r] bf16 or FP8 E4M3 (fp8). Needs
// d % 16 == 0 with d in {16, 32} or 64 <= d <= 256, r % 16 == 0 with
// 16 <= r <= 128, and project_stages(d, r, 2) >= 2.
int project_stages(int d, int r, long long ntiles);
cudaError_t launch_project(const LaunchCtx& ctx, const uint16_t* x, const uint16_t* P, void* y, bool fp8, int batch,
                           int T, int H, int d, int r, int nbases, int t0, int n, unsigned* status);
// cen [batch, ceil(T / blk), hkv, r] bf16 += kt rows t0 .. t0+n-1 of every
// sequence, in position order, rounding to bf16 after every add.
cudaError_t launch_centroid_update(const LaunchCtx& ctx, const uint16_t* kt, uint16_t* cen, int batch, int T, int hkv,
                                   int r, int blk, int t0, int n);

AttnPlan plan_attn(int nb, int hkv, int G, int B, int d, int num_sms);

// pm/pl: [units, smax, G] fp32, po: [units, smax, G, d] fp32, counters:
// [units] uint32, zero on entry and left zero. slots (optional): page table
// [nb, T] of pool rows (k/v then [nslots, hkv, d]); entries outside
// [0, nslots) are skipped and flag LSA_DEV_BAD_INDEX.
cudaError_t launch_attn(const LaunchCtx& ctx, const AttnPlan& plan, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const int32_t* idx, int B, float scale, uint16_t* out, float* pm, float* pl,
                        float* po, unsigned* counters, int nb, int hq, int hkv, int d, int T,
                        long long kv_bstride_rows, unsigned* status, const int32_t* slots = nullptr,
                        long long nslots = 0);

// Prefill indexer plan: sample stride, selection constants and the byte
// offsets of its buffers inside the caller's workspace region.
struct PrefillPlan {
    int nq_pad;              // nq rounded up to the 128-row tile
    long long rows;          // nq * hkv output rows
    int S;                   // sample stride (key columns)
    int kth;                 // rank of the sampled threshold
    int cap;                 // candidate capacity per row
    bool sample;             // some row may need a threshold (T > cap)
    int ncol_sample;         // 256-column tiles of the sample matrix
    long long ld_samp;       // sample row stride (floats)
    int stages;              // TMA pipeline stages of the score GEMM
    int a_slots;             // query tiles in flight in the score GEMM (1 or 2)
    int gemm_smem;           // dynamic shared memory of the score GEMM
    size_t off_qb, off_samp, off_thr, off_cnt, off_cand, bytes;
};

PrefillPlan plan_prefill(int hq, int hkv, int r, int T, int nq, int B);

// idx [nq, hkv, B]; ws: the plan's region (256-byte aligned, no initial value).
cudaError_t launch_prefill_index(const LaunchCtx& ctx, const PrefillPlan& P, const uint16_t* qt, const uint16_t* kt,
                                 int hq, int hkv, int r, int T, int nq, int q_start, int B, int32_t* idx, uint8_t* ws,
                                 unsigned* status);

}  // namespace lsa
