// Gather-free indexed attention (split over the index set) and the split combine.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Key
// contributions and Fig. 1: the query heads of a KV head share that head's
// index set S, and attention reads the selected K/V rows in place from the
// standard GQA cache [T, hkv, d] (no gather copy into a dense buffer). Fig. 2b
// and Fig. 6 are the pages' evidence that the gather copy is the cost to avoid.
//
// One CTA handles one (sequence, KV head, split): a slice of S. Selected rows
// are staged into shared memory with 16-byte cp.async (double buffered, tiles
// of 64 rows, zero-fill for padded entries), logits for all G heads are formed
// with fp32 FMAs, and an online softmax in the exp2 domain accumulates (m, l, o)
// per query head. Splits write fp32 partials that the combine kernel merges;
// with a single split the kernel writes the bf16 output directly.
#include <cuda_bf16.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = 4;
constexpr int kNT = 64;               // rows per tile
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
    const uint16_t* q;        // [nb, hq, D]
    const uint8_t* k;         // rows of D bf16: k + ((b * kv_bstride_rows) + t * hkv + h) * D * 2
    const uint8_t* v;
    const int32_t* idx;       // [nb, hkv, B]
    uint16_t* out;            // [nb, hq, D] (single split)
    float* pm;                // [nb, hq, nsw]
    float* pl;
    float* po;                // [nb, hq, nsw, D]
    long long kv_bstride_rows;   // T * hkv for decode, 0 for prefill (one shared cache)
    int hq, hkv, T, B;
    int rpc;                  // index-set entries per CTA (multiple of kNT)
    int nsw;                  // partial slots per head = splits * warps per head
    float qscale;             // scale * log2(e)
    unsigned* status;
    unsigned long long* counters;   // [nb, hkv] finished-split counters (zero between launches)
    int splits;
};

// Swizzled position of 16-byte chunk c of tile row j: XOR bits 1..2 of the chunk
// with the row, so that the 8 lanes of a shared-memory phase (4 rows x 2 column
// halves in the logit loop) and the 32 lanes of a value-row read hit distinct
// banks.
__device__ __forceinline__ int swz(int j, int c) { return c ^ ((j & 3) << 1); }

template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const AttnArgs a) {
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    constexpr int WPH = G >= kAttnWarps ? 1 : kAttnWarps / G;   // warps per head
    constexpr int HPW = G >= kAttnWarps ? G / kAttnWarps : 1;   // heads per warp
    constexpr int DPL = D / 32;                // output dims per lane
    constexpr int RPW = kNT / WPH;             // tile rows per warp (softmax/PV)

    extern __shared__ __align__(128) uint8_t smem[];
    const int nstages = a.rpc > kNT ? 2 : 1;
    uint8_t* kv_s = smem;                                          // [nstages][2][kNT][D] bf16
    float* qs = reinterpret_cast<float*>(smem + nstages * 2 * kNT * D * 2);   // [G][D]
    float* ps = qs + G * D;                                        // [G][kNT]
    int* rows_s = reinterpret_cast<int*>(ps + G * kNT);            // [rpc]

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int e0 = split * a.rpc;
    const int e1 = min(a.B, e0 + a.rpc);
    const int nrows = max(0, e1 - e0);
    const int ntiles = (nrows + kNT - 1) / kNT;

    // stage the slice of the index set (validated) and the scaled queries
    const int32_t* ib = a.idx + ((size_t)b * a.hkv + h) * a.B + e0;
    for (int i = tid; i < ntiles * kNT; i += kAttnThreads) {
        int t = -1;
        if (i < nrows) {
            t = ib[i];
            if (t < -1 || t >= a.T) {
                set_status(a.status, kStatusBadIndex);
                t = -1;
            }
        }
        rows_s[i] = t;
    }
    const uint16_t* qb = a.q + ((size_t)b * a.hq + (size_t)h * G) * D;
    for (int i = tid; i < G * D; i += kAttnThreads)
        qs[i] = __uint_as_float(((uint32_t)qb[i]) << 16) * a.qscale;
    __syncthreads();

    const size_t row_bytes = (size_t)D * 2;
    const uint8_t* kbase = a.k + ((size_t)b * a.kv_bstride_rows + h) * row_bytes;
    const uint8_t* vbase = a.v + ((size_t)b * a.kv_bstride_rows + h) * row_bytes;
    const size_t tstride = (size_t)a.hkv * row_bytes;

    auto load_tile = [&](int tt, int st) {
        uint8_t* ks = kv_s + (size_t)(st * 2 + 0) * kNT * row_bytes;
        uint8_t* vs = kv_s + (size_t)(st * 2 + 1) * kNT * row_bytes;
        for (int id = tid; id < kNT * CPR; id += kAttnThreads) {
            const int j = id / CPR, c = id - j * CPR;
            const int t = rows_s[tt * kNT + j];
            const size_t off = t >= 0 ? (size_t)t * tstride + c * 16 : 0;
            const uint32_t n = t >= 0 ? 16u : 0u;
            const int pc = swz(j, c);
            cp_async16(ks + j * row_bytes + pc * 16, kbase + off, n);
            cp_async16(vs + j * row_bytes + pc * 16, vbase + off, n);
        }
        cp_async_commit();
    };

    // per-warp online-softmax state: heads g = (warp % G) + 4 * hh (G >= 4) or
    // g = warp % G with row subset ws = warp / G (G < 4)
    const int ws = G >= kAttnWarps ? 0 : warp / G;
    float m_st[HPW], l_st[HPW], o_st[HPW][DPL];
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
        m_st[hh] = -INFINITY;
        l_st[hh] = 0.f;
#pragma unroll
        for (int k = 0; k < DPL; ++k) o_st[hh][k] = 0.f;
    }

    if (ntiles > 0) load_tile(0, 0);
    for (int tt = 0; tt < ntiles; ++tt) {
        const int st = tt & 1;
        if (tt + 1 < ntiles) {
            load_tile(tt + 1, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint8_t* ks = kv_s + (size_t)(st * 2 + 0) * kNT * row_bytes;
        const uint8_t* vs = kv_s + (size_t)(st * 2 + 1) * kNT * row_bytes;

        // logits: thread -> (row j, column half); all G heads at once
        {
            const int j = tid >> 1, half = tid & 1;
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = 0.f;
#pragma unroll 4
            for (int i = 0; i < CPR / 2; ++i) {
                const int c = 2 * i + half;
                const uint4 w = *reinterpret_cast<const uint4*>(ks + j * row_bytes + swz(j, c) * 16);
                const float k0 = bf16lo(w.x), k1 = bf16hi(w.x), k2 = bf16lo(w.y), k3 = bf16hi(w.y);
                const float k4 = bf16lo(w.z), k5 = bf16hi(w.z), k6 = bf16lo(w.w), k7 = bf16hi(w.w);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 qa = *reinterpret_cast<const float4*>(qs + g * D + c * 8);
                    const float4 qc = *reinterpret_cast<const float4*>(qs + g * D + c * 8 + 4);
                    float s = acc[g];
                    s = fmaf(qa.x, k0, s);
                    s = fmaf(qa.y, k1, s);
                    s = fmaf(qa.z, k2, s);
                    s = fmaf(qa.w, k3, s);
                    s = fmaf(qc.x, k4, s);
                    s = fmaf(qc.y, k5, s);
                    s = fmaf(qc.z, k6, s);
                    s = fmaf(qc.w, k7, s);
                    acc[g] = s;
                }
            }
            const bool valid = rows_s[tt * kNT + j] >= 0;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float s = acc[g] + __shfl_xor_sync(0xffffffffu, acc[g], 1);
                if ((g & 1) == half) ps[g * kNT + j] = valid ? s : -INFINITY;
            }
        }
        __syncthreads();

        // online softmax + P.V per (warp, head)
#pragma unroll
        for (int hh = 0; hh < HPW; ++hh) {
            const int g = G >= kAttnWarps ? warp + kAttnWarps * hh : warp % G;
            float* pg = ps + g * kNT;
            float tmax = -INFINITY;
            for (int r = lane; r < RPW; r += 32) tmax = fmaxf(tmax, pg[ws + WPH * r]);
            tmax = warp_max(tmax);
            const float m_new = fmaxf(m_st[hh], tmax);
            if (m_new == -INFINITY) continue;      // nothing valid yet (warp-uniform)
            const float alpha = exp2f(m_st[hh] - m_new);
            float lsum = 0.f;
            for (int r = lane; r < RPW; r += 32) {
                const int j = ws + WPH * r;
                const float e = exp2f(pg[j] - m_new);
                pg[j] = e;
                lsum += e;
            }
            __syncwarp();
            l_st[hh] = l_st[hh] * alpha + lsum;
#pragma unroll
            for (int k = 0; k < DPL; ++k) o_st[hh][k] *= alpha;
            m_st[hh] = m_new;
#pragma unroll 4
            for (int r = 0; r < RPW; ++r) {
                const int j = ws + WPH * r;
                const float e = pg[j];
                const int byte = lane * DPL * 2;
                const uint8_t* vrow = vs + j * row_bytes + swz(j, byte >> 4) * 16 + (byte & 15);
                if (DPL == 2) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(vrow);
                    o_st[hh][0] = fmaf(e, bf16lo(w), o_st[hh][0]);
                    o_st[hh][1] = fmaf(e, bf16hi(w), o_st[hh][1]);
                } else if (DPL == 4) {
                    const uint2 w = *reinterpret_cast<const uint2*>(vrow);
                    o_st[hh][0] = fmaf(e, bf16lo(w.x), o_st[hh][0]);
                    o_st[hh][1] = fmaf(e, bf16hi(w.x), o_st[hh][1]);
                    o_st[hh][2] = fmaf(e, bf16lo(w.y), o_st[hh][2]);
                    o_st[hh][3] = fmaf(e, bf16hi(w.y), o_st[hh][3]);
                } else {
                    const uint4 w = *reinterpret_cast<const uint4*>(vrow);
                    o_st[hh][0] = fmaf(e, bf16lo(w.x), o_st[hh][0]);
                    o_st[hh][1] = fmaf(e, bf16hi(w.x), o_st[hh][1]);
                    o_st[hh][2] = fmaf(e, bf16lo(w.y), o_st[hh][2]);
                    o_st[hh][3] = fmaf(e, bf16hi(w.y), o_st[hh][3]);
                    o_st[hh][4] = fmaf(e, bf16lo(w.z), o_st[hh][4]);
                    o_st[hh][5] = fmaf(e, bf16hi(w.z), o_st[hh][5]);
                    o_st[hh][6] = fmaf(e, bf16lo(w.w), o_st[hh][6]);
                    o_st[hh][7] = fmaf(e, bf16hi(w.w), o_st[hh][7]);
                }
            }
        }
        __syncthreads();
    }

    // write partial (m, l, o) or, with one slot per head, the final output
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
        const int g = G >= kAttnWarps ? warp + kAttnWarps * hh : warp % G;
        const int qh = h * G + g;
        const float l = warp_sum(l_st[hh]);
        if (a.nsw == 1) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint16_t* o = a.out + ((size_t)b * a.hq + qh) * D + lane * DPL;
#pragma unroll
            for (int k = 0; k < DPL; ++k) o[k] = f2bf(o_st[hh][k] * inv);
        } else {
            const int slot = split * WPH + ws;
            const size_t pi = ((size_t)b * a.hq + qh) * a.nsw + slot;
            if (lane == 0) {
                a.pm[pi] = m_st[hh];
                a.pl[pi] = l;
            }
            float* po = a.po + pi * D + lane * DPL;
#pragma unroll
            for (int k = 0; k < DPL; ++k) po[k] = o_st[hh][k];
        }
    }
    if (a.nsw == 1) return;

    // The last CTA of this (row, KV head) to finish merges every slot of its
    // G query heads (threadfence-reduction pattern; the counter is left at 0).
    __threadfence();
    __syncthreads();
    __shared__ int is_last;
    if (tid == 0) {
        unsigned long long* cnt = a.counters + (size_t)b * a.hkv + h;
        const unsigned long long old = atomicAdd(cnt, 1ull);
        is_last = old + 1 == (unsigned long long)a.splits;
        if (is_last) atomicExch(cnt, 0ull);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int g = warp; g < G; g += kAttnWarps) {
        const size_t w = (size_t)b * a.hq + h * G + g;
        const float* m = a.pm + w * a.nsw;
        const float* l = a.pl + w * a.nsw;
        float M = -INFINITY;
        for (int s = lane; s < a.nsw; s += 32) M = fmaxf(M, __ldcg(m + s));
        M = warp_max(M);
        float acc[DPL];
#pragma unroll
        for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
        float L = 0.f;
        if (M != -INFINITY) {
            // lanes own slots for the weights; the slot loop below keeps eight
            // independent partial-row loads in flight per lane
            for (int s0 = 0; s0 < a.nsw; s0 += 32) {
                const int s = s0 + lane;
                float wgt = 0.f;
                if (s < a.nsw) {
                    const float ms = __ldcg(m + s);
                    if (ms != -INFINITY) {
                        wgt = exp2f(ms - M);
                        L = fmaf(wgt, __ldcg(l + s), L);
                    }
                }
                const int cnt = min(32, a.nsw - s0);
                for (int j0 = 0; j0 < cnt; j0 += 8) {
                    float vals[8][DPL];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float* o = a.po + (w * a.nsw + s0 + j0 + u) * D + lane * DPL;
#pragma unroll
                        for (int k = 0; k < DPL; ++k) vals[u][k] = j0 + u < cnt ? __ldcg(o + k) : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float wu = __shfl_sync(0xffffffffu, wgt, (j0 + u) & 31);
#pragma unroll
                        for (int k = 0; k < DPL; ++k) acc[k] = fmaf(wu, vals[u][k], acc[k]);
                    }
                }
            }
            L = warp_sum(L);
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        uint16_t* o = a.out + w * D + lane * DPL;
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[k] = f2bf(acc[k] * inv);
    }
}

int attn_stages(int rpc) { return rpc > kNT ? 2 : 1; }

size_t attn_smem_bytes(int D, int G, int rpc) {
    return (size_t)attn_stages(rpc) * 2 * kNT * D * 2 + (size_t)G * D * 4 + (size_t)G * kNT * 4 + (size_t)rpc * 4;
}

template <int D, int G>
cudaError_t launch_attn_t(const LaunchCtx& ctx, const AttnArgs& a, int splits, int nb) {
    const size_t smem = attn_smem_bytes(D, G, a.rpc);
    auto kern = attn_kernel<D, G>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)splits, (unsigned)a.hkv, (unsigned)nb);
    kern<<<grid, kAttnThreads, smem, ctx.stream>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_attn_d(const LaunchCtx& ctx, const AttnArgs& a, int G, int splits, int nb) {
    switch (G) {
        case 1: return launch_attn_t<D, 1>(ctx, a, splits, nb);
        case 2: return launch_attn_t<D, 2>(ctx, a, splits, nb);
        case 4: return launch_attn_t<D, 4>(ctx, a, splits, nb);
        case 8: return launch_attn_t<D, 8>(ctx, a, splits, nb);
        case 16: return launch_attn_t<D, 16>(ctx, a, splits, nb);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

AttnPlan plan_attn(int nb, int hkv, int G, int B, int num_sms) {
    // Largest slice (a multiple of one 64-row tile, at most 1024 rows) that
    // still gives about six CTAs per SM; one-tile slices keep a single stage.
    AttnPlan p{};
    const long long units = (long long)nb * hkv;
    const long long target = 6ll * num_sms;
    int rpc = kNT;
    while (rpc < 1024 && units * ((B + 2 * rpc - 1) / (2 * rpc)) >= target) rpc *= 2;
    p.rpc = rpc;
    p.splits = (B + rpc - 1) / rpc;
    const int wph = G >= kAttnWarps ? 1 : kAttnWarps / G;
    p.nsw = p.splits * wph;
    return p;
}

cudaError_t launch_attn(const LaunchCtx& ctx, const AttnPlan& plan, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const int32_t* idx, int B, float scale, uint16_t* out, float* pm, float* pl,
                        float* po, unsigned long long* counters, int nb, int hq, int hkv, int d, int T,
                        long long kv_bstride_rows, unsigned* status) {
    AttnArgs a{};
    a.q = q;
    a.k = reinterpret_cast<const uint8_t*>(k);
    a.v = reinterpret_cast<const uint8_t*>(v);
    a.idx = idx;
    a.out = out;
    a.pm = pm;
    a.pl = pl;
    a.po = po;
    a.kv_bstride_rows = kv_bstride_rows;
    a.hq = hq;
    a.hkv = hkv;
    a.T = T;
    a.B = B;
    a.rpc = plan.rpc;
    a.nsw = plan.nsw;
    a.qscale = scale * kLog2e;
    a.status = status;
    a.counters = counters;
    a.splits = plan.splits;
    const int G = hq / hkv;
    switch (d) {
        case 64: return launch_attn_d<64>(ctx, a, G, plan.splits, nb);
        case 128: return launch_attn_d<128>(ctx, a, G, plan.splits, nb);
        case 256: return launch_attn_d<256>(ctx, a, G, plan.splits, nb);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
