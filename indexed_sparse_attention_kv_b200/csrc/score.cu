// Candidate scoring kernels: flat streaming scorer, fine (candidate-list)
// scorer for coarse-to-fine mode, and block centroids.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Fig. 1:
// for each KV head, the mean of its query group scores every row of a
// projected-key cache [T, hkv, r]. The scorer is an HBM stream: every byte of
// the projected-key cache is read once, through 1-D TMA bulk copies into a
// multi-stage shared-memory ring, and reduced with fp32 FMAs.
#include <cuda_bf16.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kScoreStages = 4;
constexpr int kChunkTarget = 16384;   // bytes per pipeline stage (approximate)

struct ScoreArgs {
    const uint16_t* qt;    // [batch, hq, r]
    const uint8_t* kt;     // [batch, n, hkv, r] bf16 (or FP8 E4M3 for the FP8 scorer)
    float* out;            // [batch, hkv, n]
    int hq, hkv, n, G;
    int tok_per_chunk;     // tokens per stage, multiple of the tokens per warp pass
    int chunks_per_batch;
    int ctas_per_batch;
    int mode;              // 0: group sum, 1: group mean
    int g_pow2;
    float inv_g;
    unsigned* status;
    long long wait_limit;
    uint32_t* ghist;       // optional [batch, hkv, 2048] key histogram (fast path only)
};

__device__ __forceinline__ float finalize_score(float acc, const ScoreArgs& a) {
    if (a.mode == 0) return acc;
    return a.g_pow2 ? acc * a.inv_g : __fdiv_rn(acc, (float)a.G);
}

// Two OCP FP8 E4M3 values (element 0 in the low byte) -> two floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// 16 E4M3 values . q[0..16), fp32 accumulation in two interleaved chains (even
// and odd channels, summed at the end) so that consecutive FMAs do not wait on
// each other.
__device__ __forceinline__ float dot16_e4m3(const uint4 w, const float* q) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f0 = e4m3x2_to_float2(ws[i]);
        const float2 f1 = e4m3x2_to_float2(ws[i] >> 16);
        acc0 = fmaf(q[4 * i + 0], f0.x, acc0);
        acc1 = fmaf(q[4 * i + 1], f0.y, acc1);
        acc0 = fmaf(q[4 * i + 2], f1.x, acc0);
        acc1 = fmaf(q[4 * i + 3], f1.y, acc1);
    }
    return acc0 + acc1;
}

__device__ __forceinline__ float dot8(const uint4 w, const float* q) {
    float acc = 0.f;
    acc = fmaf(q[0], bf16lo(w.x), acc);
    acc = fmaf(q[1], bf16hi(w.x), acc);
    acc = fmaf(q[2], bf16lo(w.y), acc);
    acc = fmaf(q[3], bf16hi(w.y), acc);
    acc = fmaf(q[4], bf16lo(w.z), acc);
    acc = fmaf(q[5], bf16hi(w.z), acc);
    acc = fmaf(q[6], bf16lo(w.w), acc);
    acc = fmaf(q[7], bf16hi(w.w), acc);
    return acc;
}

// One CTA streams a contiguous range of chunks of one sequence. A chunk is
// tok_per_chunk whole tokens (all hkv heads, r channels each). A warp pass
// covers TPW consecutive tokens of one head: LPR = r/8 lanes per row, each lane
// 16 bytes, so a pass reads TPW rows and writes TPW consecutive scores.
template <int R, bool FIXED_HEAD>
__global__ void __launch_bounds__(kScoreThreads) score_flat_kernel(const ScoreArgs a) {
    constexpr int LPR = R / 8;
    constexpr int TPW = 32 / LPR;
    extern __shared__ __align__(128) uint8_t smem[];
    const int hkv = a.hkv;
    const int row_bytes = R * 2;
    const int token_bytes = hkv * row_bytes;
    const int chunk_bytes = a.tok_per_chunk * token_bytes;
    uint8_t* stages = smem;
    float* qbar = reinterpret_cast<float*>(smem + kScoreStages * chunk_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(qbar + hkv * R);

    const int b = blockIdx.y;
    const int c0 = (int)((long long)blockIdx.x * a.chunks_per_batch / a.ctas_per_batch);
    const int c1 = (int)((long long)(blockIdx.x + 1) * a.chunks_per_batch / a.ctas_per_batch);
    const int nch = c1 - c0;
    const uint8_t* kt_b = a.kt + (size_t)b * a.n * token_bytes;

    // Group-sum query of every KV head (fp32; exact for integer-valued bf16).
    for (int e = threadIdx.x; e < hkv * R; e += kScoreThreads) {
        const int h = e / R, j = e - h * R;
        const uint16_t* src = a.qt + ((size_t)b * a.hq + (size_t)h * a.G) * R + j;
        float s = 0.f;
        for (int g = 0; g < a.G; ++g) s += __uint_as_float(((uint32_t)src[(size_t)g * R]) << 16);
        qbar[e] = s;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kScoreStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int i) {
        const int t0 = (c0 + i) * a.tok_per_chunk;
        const int ntok = min(a.tok_per_chunk, a.n - t0);
        const uint32_t bytes = (uint32_t)(ntok * token_bytes);
        uint64_t* bar = &bars[i % kScoreStages];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(stages + (i % kScoreStages) * chunk_bytes, kt_b + (size_t)t0 * token_bytes, bytes, bar);
    };
    if (threadIdx.x == 0) {
        const int npro = min(kScoreStages, nch);
        for (int i = 0; i < npro; ++i) issue(i);
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR;      // token within the warp pass
    const int cpart = lane % LPR;    // 16-byte column chunk of the row
    float qreg[8];
    if (FIXED_HEAD) {
        const float* qs = qbar + (warp % hkv) * R + cpart * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) qreg[k] = qs[k];
    }
    const int items = hkv * (a.tok_per_chunk / TPW);
    float* out_b = a.out + (size_t)b * hkv * a.n;

    int i = 0;
    bool timed_out = false;
    for (; i < nch; ++i) {
        const int s = i % kScoreStages;
        const bool ready = mbar_wait_bounded(&bars[s], (uint32_t)((i / kScoreStages) & 1), a.wait_limit);
        if (!__syncthreads_and(ready)) {
            timed_out = true;
            break;
        }
        const int t0 = (c0 + i) * a.tok_per_chunk;
        const int ntok = min(a.tok_per_chunk, a.n - t0);
        const uint8_t* st = stages + s * chunk_bytes;
        for (int item = warp; item < items; item += kScoreWarps) {
            const int h = FIXED_HEAD ? (warp % hkv) : (item % hkv);
            const int tl = (item / hkv) * TPW + sub;
            float acc = 0.f;
            if (tl < ntok) {
                const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)tl * token_bytes + h * row_bytes + cpart * 16);
                if (FIXED_HEAD) {
                    acc = dot8(w, qreg);
                } else {
                    float qv[8];
                    const float* qs = qbar + h * R + cpart * 8;
#pragma unroll
                    for (int k = 0; k < 8; ++k) qv[k] = qs[k];
                    acc = dot8(w, qv);
                }
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (cpart == 0 && tl < ntok) out_b[(size_t)h * a.n + t0 + tl] = finalize_score(acc, a);
        }
        __syncthreads();
        if (threadIdx.x == 0 && i + kScoreStages < nch) issue(i + kScoreStages);
    }
    if (timed_out) {
        // Leave no bulk copy in flight into this CTA's shared memory.
        if (threadIdx.x == 0) {
            set_status(a.status, kStatusTimeout);
            const int issued = min(nch, i + kScoreStages);
            for (int j = i; j < issued; ++j)
                mbar_wait_bounded(&bars[j % kScoreStages], (uint32_t)((j / kScoreStages) & 1), kDrainNs);
        }
        __syncthreads();
    }
}

// Fine scorer for coarse-to-fine mode: candidate c of (b, h) is token
// blk_idx[b,h,c / blk] * blk + c % blk; scores go to out[b, h, c], NaN for a
// padded block or a token past T. Direct 16-byte loads (rows are scattered).
struct FineArgs {
    const uint16_t* qt;
    const uint8_t* kt;
    const int32_t* blk_idx;   // [batch, hkv, keep]
    float* out;               // [batch, hkv, keep * blk]
    int hq, hkv, T, G, blk, keep, ncand;
};

template <int R>
__global__ void __launch_bounds__(256) score_fine_kernel(const FineArgs a) {
    constexpr int LPR = R / 8;
    constexpr int TPW = 32 / LPR;
    const int h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, cpart = lane % LPR;
    float q[8];
    {
        const uint16_t* src = a.qt + ((size_t)b * a.hq + (size_t)h * a.G) * R + cpart * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) q[k] = 0.f;
        for (int g = 0; g < a.G; ++g)
#pragma unroll
            for (int k = 0; k < 8; ++k) q[k] += __uint_as_float(((uint32_t)src[(size_t)g * R + k]) << 16);
    }
    pdl_launch_dependents();
    pdl_wait();   // the kept block ids come from the previous kernel
    const int32_t* bi = a.blk_idx + ((size_t)b * a.hkv + h) * a.keep;
    float* out = a.out + ((size_t)b * a.hkv + h) * a.ncand;
    const size_t row_stride = (size_t)a.hkv * R * 2;
    const uint8_t* base = a.kt + (size_t)b * a.T * row_stride + (size_t)h * R * 2 + cpart * 16;
    const int per_cta = (a.ncand + gridDim.x - 1) / gridDim.x;
    const int cbeg = blockIdx.x * per_cta, cend = min(a.ncand, cbeg + per_cta);
    for (int c_base = cbeg + warp * TPW; c_base < cend; c_base += 8 * TPW) {
        const int c = c_base + sub;
        bool valid = false;
        float acc = 0.f;
        if (c < cend) {
            const int j = c / a.blk;
            const int blkid = bi[j];
            const long long pos = (long long)blkid * a.blk + (c - j * a.blk);
            valid = blkid >= 0 && pos < a.T;
            if (valid) acc = dot8(ldg_stream16(base + (size_t)pos * row_stride), q);
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (cpart == 0 && c < cend) out[c] = valid ? acc : __int_as_float(0x7fc00000);
    }
}

// Block centroids: c[b, j, h, :] = sum over the block's tokens of kt[b, t, h, :].
// One CTA per (block, sequence); thread i owns 8 consecutive channels of the
// [hkv * r] token row.
__global__ void __launch_bounds__(512) centroid_kernel(const uint8_t* kt, uint16_t* cen, int T, int blk, int row_elems,
                                                        int nblk) {
    const int j = blockIdx.x, b = blockIdx.y;
    const int i = threadIdx.x;
    if (i * 8 >= row_elems) return;
    const size_t row_bytes = (size_t)row_elems * 2;
    const uint8_t* src = kt + ((size_t)b * T + (size_t)j * blk) * row_bytes + (size_t)i * 16;
    const int ntok = min(blk, T - j * blk);
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    for (int t = 0; t < ntok; ++t) {
        const uint4 w = ldg_stream16(src + (size_t)t * row_bytes);
        acc[0] += bf16lo(w.x); acc[1] += bf16hi(w.x);
        acc[2] += bf16lo(w.y); acc[3] += bf16hi(w.y);
        acc[4] += bf16lo(w.z); acc[5] += bf16hi(w.z);
        acc[6] += bf16lo(w.w); acc[7] += bf16hi(w.w);
    }
    uint4 o;
    o.x = (uint32_t)f2bf(acc[0]) | ((uint32_t)f2bf(acc[1]) << 16);
    o.y = (uint32_t)f2bf(acc[2]) | ((uint32_t)f2bf(acc[3]) << 16);
    o.z = (uint32_t)f2bf(acc[4]) | ((uint32_t)f2bf(acc[5]) << 16);
    o.w = (uint32_t)f2bf(acc[6]) | ((uint32_t)f2bf(acc[7]) << 16);
    *reinterpret_cast<uint4*>(cen + ((size_t)b * nblk + j) * row_elems + (size_t)i * 8) = o;
}

// Fast path for r = 64 and hkv in {4, 8, 16, 32}: warp-specialised pipeline.
// One producer warp streams 16 KiB chunks through a STAGES-deep ring of TMA
// bulk copies (full barriers carry the byte count, empty barriers collect one
// arrival per consumer warp). A consumer warp pass covers 4 tokens x 4 heads:
// lane = (head-in-quad, token, half-row); each lane keeps its 32 group-sum
// query values in registers (rotated so that the 8 lanes of a shared-memory
// phase read 8 distinct 16-byte bank groups), does 32 FMAs, and one shuffle
// joins the two halves of a row.
// HIST: also count, per KV head, the top 11 bits of every score's order key
// (the first radix digit of the top-B selection) in a shared-memory histogram
// of 16-bit counters, added to a global per-(sequence, head) histogram at the
// end; that saves the selection a full pass over the scores.
constexpr int kQConsumers = 8;
constexpr int kQThreads = (kQConsumers + 1) * 32;
constexpr int kQChunk = 16384;
constexpr int kHistBins = 2048;

// FP8: the projected keys are OCP FP8 E4M3 (64 bytes per head row) instead of
// bf16 (128 bytes); every lane then reads 32 channels as two 16-byte words.
template <int STAGES, bool HIST, bool FP8>
__global__ void __launch_bounds__(kQThreads, 2) score_q64_kernel(const ScoreArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int hkv = a.hkv;
    constexpr int kHeadBytes = FP8 ? 64 : 128;
    const int token_bytes = hkv * kHeadBytes;
    const int tok = a.tok_per_chunk;
    uint8_t* stages = smem;
    float* qbar = reinterpret_cast<float*>(smem + STAGES * kQChunk);
    uint32_t* hs = reinterpret_cast<uint32_t*>(qbar + hkv * 64);          // [hkv][kHistBins / 2] (HIST)
    uint64_t* full = reinterpret_cast<uint64_t*>(hs + (HIST ? hkv * kHistBins / 2 : 0));
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);

    const int b = blockIdx.y;
    const int c0 = (int)((long long)blockIdx.x * a.chunks_per_batch / a.ctas_per_batch);
    const int c1 = (int)((long long)(blockIdx.x + 1) * a.chunks_per_batch / a.ctas_per_batch);
    const int nch = c1 - c0;
    const uint8_t* kt_b = a.kt + (size_t)b * a.n * token_bytes;

    for (int e = threadIdx.x; e < hkv * 64; e += kQThreads) {
        const int h = e >> 6, j = e & 63;
        const uint16_t* src = a.qt + ((size_t)b * a.hq + (size_t)h * a.G) * 64 + j;
        float s = 0.f;
        for (int g = 0; g < a.G; ++g) s += __uint_as_float(((uint32_t)src[(size_t)g * 64]) << 16);
        qbar[e] = s;
    }
    if (HIST)
        for (int e = threadIdx.x; e < hkv * kHistBins / 2; e += kQThreads) hs[e] = 0u;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();   // the selection kernel may start its prologue
    int issued = 0;            // bulk copies issued (producer lane)
    if (warp == kQConsumers) {
        if (lane == 0) {
            const uint64_t stream_pol = policy_evict_first();   // read-once stream: keep it out of L2's way
            for (int i = 0; i < nch; ++i) {
                const int s = i % STAGES;
                if (i >= STAGES &&
                    !mbar_wait_bounded(&empty[s], (uint32_t)(((i / STAGES) - 1) & 1), a.wait_limit, abort_flag)) {
                    *abort_flag = 1;
                    break;
                }
                const int t0 = (c0 + i) * tok;
                const int ntok = min(tok, a.n - t0);
                const uint32_t bytes = (uint32_t)(ntok * token_bytes);
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s_hint(stages + s * kQChunk, kt_b + (size_t)t0 * token_bytes, bytes, &full[s], stream_pol);
                issued = i + 1;
            }
        }
    } else {
        const int quads = hkv >> 2;
        const int q = warp % quads;
        const int wpq = kQConsumers / quads;
        const int half = lane & 1, tsub = (lane >> 1) & 3, hl = lane >> 3;
        const int head = q * 4 + hl;
        float qv[32];
        if (FP8) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float* src = qbar + head * 64 + half * 32 + ((k + tsub) & 1) * 16;
#pragma unroll
                for (int e = 0; e < 16; ++e) qv[k * 16 + e] = src[e];
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float* src = qbar + head * 64 + half * 32 + ((k + tsub) & 3) * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) qv[k * 8 + e] = src[e];
            }
        }
        float* out_h = a.out + ((size_t)b * hkv + head) * a.n;
        const uint64_t keep_pol = policy_evict_last();   // the top-B selection re-reads the scores
        uint32_t* hs_h = hs + head * (kHistBins / 2);
        for (int i = 0; i < nch; ++i) {
            const int s = i % STAGES;
            if (!mbar_wait_bounded(&full[s], (uint32_t)((i / STAGES) & 1), a.wait_limit, abort_flag)) {
                *abort_flag = 1;
                break;
            }
            const int t0 = (c0 + i) * tok;
            const int ntok = min(tok, a.n - t0);
            const uint8_t* st = stages + s * kQChunk + head * kHeadBytes + half * (kHeadBytes / 2);
            for (int tg = warp / quads; tg * 4 < ntok; tg += wpq) {
                const int t = tg * 4 + tsub;
                float acc0 = 0.f, acc1 = 0.f;
                if (t < ntok) {
                    const uint8_t* row = st + (size_t)t * token_bytes;
                    if (FP8) {
                        const uint4 w0 = *reinterpret_cast<const uint4*>(row + ((0 + tsub) & 1) * 16);
                        const uint4 w1 = *reinterpret_cast<const uint4*>(row + ((1 + tsub) & 1) * 16);
                        acc0 = dot16_e4m3(w0, qv + 0);
                        acc1 = dot16_e4m3(w1, qv + 16);
                    } else {
                        const uint4 w0 = *reinterpret_cast<const uint4*>(row + ((0 + tsub) & 3) * 16);
                        const uint4 w1 = *reinterpret_cast<const uint4*>(row + ((1 + tsub) & 3) * 16);
                        const uint4 w2 = *reinterpret_cast<const uint4*>(row + ((2 + tsub) & 3) * 16);
                        const uint4 w3 = *reinterpret_cast<const uint4*>(row + ((3 + tsub) & 3) * 16);
                        acc0 = dot8(w0, qv + 0);
                        acc1 = dot8(w1, qv + 8);
                        acc0 += dot8(w2, qv + 16);
                        acc1 += dot8(w3, qv + 24);
                    }
                }
                float acc = acc0 + acc1;
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (half == 0 && t < ntok) {
                    const float v = finalize_score(acc, a);
                    st_hint(out_h + t0 + t, v, keep_pol);
                    if (HIST) {
                        const uint32_t key = score_key(v);
                        if (key) atomicAdd(&hs_h[key >> 22], 1u << (((key >> 21) & 1u) * 16));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    __syncthreads();
    if (*abort_flag) {
        // Every role has stopped, and an abort from any of them is visible
        // here. Leave no bulk copy in flight into this CTA's shared memory:
        // each stage has at most one outstanding phase, its last issued one.
        if (warp == kQConsumers && lane == 0) {
            set_status(a.status, kStatusTimeout);
            for (int s = 0; s < STAGES && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / STAGES) * STAGES;
                mbar_wait_bounded(&full[s], (uint32_t)((last / STAGES) & 1), kDrainNs);
            }
        }
        __syncthreads();
    }
    if (HIST) {
        uint32_t* gh = a.ghist + (size_t)b * hkv * kHistBins;
        for (int e = threadIdx.x; e < hkv * kHistBins / 2; e += kQThreads) {
            const uint32_t v = hs[e];
            if (!v) continue;
            const int h = e / (kHistBins / 2), w = e - h * (kHistBins / 2);
            uint32_t* dst = gh + (size_t)h * kHistBins + 2 * w;
            if (v & 0xffffu) atomicAdd(dst, v & 0xffffu);
            if (v >> 16) atomicAdd(dst + 1, v >> 16);
        }
    }
}

template <int STAGES, bool HIST, bool FP8>
cudaError_t launch_q64_t(const LaunchCtx& ctx, ScoreArgs a, int batch) {
    const size_t smem = (size_t)STAGES * kQChunk + (size_t)a.hkv * 64 * 4 +
                        (HIST ? (size_t)a.hkv * kHistBins / 2 * 4 : 0) + 2 * STAGES * 8 + 16;
    auto kern = score_q64_kernel<STAGES, HIST, FP8>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cached_occupancy((const void*)kern, kQThreads, smem, &occ);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    const long long target = (long long)ctx.num_sms * occ;
    long long per_b = (target + batch - 1) / batch;
    if (per_b > a.chunks_per_batch) per_b = a.chunks_per_batch;
    if (per_b < 1) per_b = 1;
    a.ctas_per_batch = (int)per_b;
    dim3 grid((unsigned)per_b, (unsigned)batch);
    kern<<<grid, kQThreads, smem, ctx.stream>>>(a);
    return cudaGetLastError();
}

// Returns whether the histogram was produced (a.ghist non-null, hkv <= 8 and at
// most 65535 tokens per CTA so that 16-bit shared counters cannot overflow).
cudaError_t launch_q64(const LaunchCtx& ctx, ScoreArgs a, int batch, bool* hist_done, bool fp8 = false) {
    const int token_bytes = a.hkv * (fp8 ? 64 : 128);
    a.tok_per_chunk = kQChunk / token_bytes;
    a.chunks_per_batch = (a.n + a.tok_per_chunk - 1) / a.tok_per_chunk;
    bool hist = a.ghist != nullptr && a.hkv <= 8;
    if (hist) {
        // the smallest grid the launcher can pick: one CTA per SM (occupancy >= 1)
        const long long min_per_b = ((long long)ctx.num_sms + batch - 1) / batch;
        const long long per_b = min_per_b < a.chunks_per_batch ? min_per_b : a.chunks_per_batch;
        const long long max_chunks = (a.chunks_per_batch + per_b - 1) / per_b;
        hist = max_chunks * a.tok_per_chunk <= 65535;
    }
    *hist_done = hist;
    if (fp8) return hist ? launch_q64_t<4, true, true>(ctx, a, batch) : launch_q64_t<6, false, true>(ctx, a, batch);
    return hist ? launch_q64_t<4, true, false>(ctx, a, batch) : launch_q64_t<6, false, false>(ctx, a, batch);
}

template <int R, bool FIXED>
cudaError_t launch_flat_t(const LaunchCtx& ctx, ScoreArgs a, int batch) {
    constexpr int LPR = R / 8;
    constexpr int TPW = 32 / LPR;
    const int token_bytes = a.hkv * R * 2;
    int tok = kChunkTarget / token_bytes;
    tok = tok < TPW ? TPW : (tok / TPW) * TPW;
    a.tok_per_chunk = tok;
    a.chunks_per_batch = (a.n + tok - 1) / tok;
    const size_t smem = (size_t)kScoreStages * tok * token_bytes + (size_t)a.hkv * R * 4 + kScoreStages * 8;
    auto kern = score_flat_kernel<R, FIXED>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cached_occupancy((const void*)kern, kScoreThreads, smem, &occ);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    const long long target = (long long)ctx.num_sms * occ;
    long long per_b = (target + batch - 1) / batch;
    if (per_b > a.chunks_per_batch) per_b = a.chunks_per_batch;
    if (per_b < 1) per_b = 1;
    a.ctas_per_batch = (int)per_b;
    dim3 grid((unsigned)per_b, (unsigned)batch);
    kern<<<grid, kScoreThreads, smem, ctx.stream>>>(a);
    return cudaGetLastError();
}

template <int R>
cudaError_t launch_flat_r(const LaunchCtx& ctx, const ScoreArgs& a, int batch) {
    const bool fixed = (kScoreWarps % a.hkv) == 0;
    return fixed ? launch_flat_t<R, true>(ctx, a, batch) : launch_flat_t<R, false>(ctx, a, batch);
}

template <int R>
cudaError_t launch_fine_r(const LaunchCtx& ctx, const FineArgs& a, int batch) {
    constexpr int TPW = 32 / (R / 8);
    // one pass per warp: its two dependent loads (block id, then the row) are
    // the whole latency chain
    const int per_cta_target = 8 * TPW;
    int ctas = (a.ncand + per_cta_target - 1) / per_cta_target;
    if (ctas < 1) ctas = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ctas, (unsigned)a.hkv, (unsigned)batch);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, score_fine_kernel<R>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score(const LaunchCtx& ctx, const uint16_t* qt, const uint16_t* kt, float* out, int batch, int hq,
                         int hkv, int r, int n, int mode, unsigned* status, uint32_t* ghist, bool* hist_done) {
    ScoreArgs a{};
    a.qt = qt;
    a.kt = reinterpret_cast<const uint8_t*>(kt);
    a.out = out;
    a.hq = hq;
    a.hkv = hkv;
    a.n = n;
    a.G = hq / hkv;
    a.mode = mode;
    a.g_pow2 = (a.G & (a.G - 1)) == 0;
    a.inv_g = 1.0f / (float)a.G;
    a.status = status;
    a.wait_limit = ctx.wait_limit;
    a.ghist = ghist;
    if (hist_done) *hist_done = false;
    bool dummy = false;
    if (r == 64 && (hkv == 4 || hkv == 8 || hkv == 16 || hkv == 32))
        return launch_q64(ctx, a, batch, hist_done ? hist_done : &dummy);
    switch (r) {
        case 16: return launch_flat_r<16>(ctx, a, batch);
        case 32: return launch_flat_r<32>(ctx, a, batch);
        case 64: return launch_flat_r<64>(ctx, a, batch);
        case 128: return launch_flat_r<128>(ctx, a, batch);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_score_fp8(const LaunchCtx& ctx, const uint16_t* qt, const uint8_t* kt, float* out, int batch,
                             int hq, int hkv, int r, int n, int mode, unsigned* status, uint32_t* ghist,
                             bool* hist_done) {
    if (hist_done) *hist_done = false;
    if (r != 64 || !(hkv == 4 || hkv == 8 || hkv == 16 || hkv == 32)) return cudaErrorInvalidValue;
    ScoreArgs a{};
    a.qt = qt;
    a.kt = kt;
    a.out = out;
    a.hq = hq;
    a.hkv = hkv;
    a.n = n;
    a.G = hq / hkv;
    a.mode = mode;
    a.g_pow2 = (a.G & (a.G - 1)) == 0;
    a.inv_g = 1.0f / (float)a.G;
    a.status = status;
    a.wait_limit = ctx.wait_limit;
    a.ghist = ghist;
    bool dummy = false;
    return launch_q64(ctx, a, batch, hist_done ? hist_done : &dummy, true);
}

cudaError_t launch_fine_score(const LaunchCtx& ctx, const uint16_t* qt, const uint16_t* kt, const int32_t* blk_idx,
                              int keep, int blk, float* out, int batch, int hq, int hkv, int r, int T) {
    FineArgs a{};
    a.qt = qt;
    a.kt = reinterpret_cast<const uint8_t*>(kt);
    a.blk_idx = blk_idx;
    a.out = out;
    a.hq = hq;
    a.hkv = hkv;
    a.T = T;
    a.G = hq / hkv;
    a.blk = blk;
    a.keep = keep;
    a.ncand = keep * blk;
    switch (r) {
        case 16: return launch_fine_r<16>(ctx, a, batch);
        case 32: return launch_fine_r<32>(ctx, a, batch);
        case 64: return launch_fine_r<64>(ctx, a, batch);
        case 128: return launch_fine_r<128>(ctx, a, batch);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_centroids(const LaunchCtx& ctx, const uint16_t* kt, int blk, uint16_t* cen, int batch, int hkv, int r,
                             int T) {
    const int row_elems = hkv * r;
    const int nblk = (T + blk - 1) / blk;
    int threads = ((row_elems / 8) + 31) / 32 * 32;
    dim3 grid((unsigned)nblk, (unsigned)batch);
    centroid_kernel<<<grid, threads, 0, ctx.stream>>>(reinterpret_cast<const uint8_t*>(kt), cen, T, blk, row_elems,
                                                      nblk);
    return cudaGetLastError();
}

}  // namespace lsa
