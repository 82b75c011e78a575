// Gather-free indexed attention: a persistent, stream-K split over the index sets.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Key
// contributions and Fig. 1: the query heads of a KV head share that head's
// index set S, and attention reads the selected K/V rows in place from the
// standard GQA cache [T, hkv, d] (no gather copy into a dense buffer). Fig. 2b
// and Fig. 6 are the pages' evidence that the gather copy is the cost to avoid.
//
// Work: unit u = (row b, KV head h) owns ceil(B / 64) tiles of 64 index-set
// entries; the tiles of all units, in unit order, are cut into P contiguous
// ranges, one per CTA (P = one wave: the SM count times the CTAs that fit).
// A CTA streams its tiles through a kStages-deep ring: the selected K and V
// rows and the unit's queries land in shared memory by 16-byte cp.async
// (zero-fill for padded entries), the index rows of the tile kStages ahead are
// read into registers one iteration early. Logits for the G heads are fp32 FMAs;
// an online softmax in the exp2 domain accumulates (m, l, o) per query head over
// the CTA's part of a unit (a segment). At a segment's end the CTA either
// writes the output (the unit lies entirely in this CTA) or a partial; the last
// CTA to finish a unit, found with a release/acquire counter, merges the unit's
// partials and leaves the counter at zero.
#include <cuda_bf16.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = 4;
constexpr int kNT = 64;               // index-set entries per tile
constexpr int kStages = 3;
constexpr int kPS = kNT + 4;          // padded logit row (conflict-free fragment reads)
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
    const uint16_t* q;        // [nb, hq, D]
    const uint8_t* k;         // row (b, t, h) at k + ((b * kv_bstride_rows) + t * hkv + h) * D * 2
    const uint8_t* v;
    const int32_t* idx;       // [nb * hkv, B]
    uint16_t* out;            // [nb, hq, D]
    float* pm;                // [units, smax, G]
    float* pl;
    float* po;                // [units, smax, G, D]
    unsigned* counters;       // [units] finished-segment counters (zero between launches)
    long long kv_bstride_rows;   // T * hkv for decode, 0 for prefill (one shared cache)
    int hq, hkv, T, B;
    int units, tiles_per_unit, ctas, smax;
    long long total_tiles;
    float qscale;             // scale * log2(e)
    unsigned* status;
};

// CTA that owns flattened tile w (ranges lo_p = p * W / P).
__device__ __forceinline__ int owner(long long w, const AttnArgs& a) {
    return (int)(((w + 1) * (long long)a.ctas - 1) / a.total_tiles);
}

// Swizzled position of 16-byte chunk c of tile row j: XOR with the row's low 3
// bits, so that the 8 row addresses of every ldmatrix phase hit 8 distinct
// 16-byte bank groups.
__device__ __forceinline__ int swz(int j, int c) { return c ^ (j & 7); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}
// D += A (16x16 bf16, row) * B (16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two fp32 -> packed bf16x2 (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D, int G>
struct AttnLayout {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kKV = kNT * kRowBytes;                 // one of K or V per stage
    static constexpr int kQ = G * D * 2;                         // the unit's queries (bf16)
    static constexpr int kStage = 2 * kKV + kQ;                  // K, V, q
    static constexpr int kP = G * (kNT + 4) * 4;                 // logits / weights (padded rows)
    static constexpr int kHead = 3 * 16 * 4;                     // running max, sum, rescale per head
    static constexpr int kRows = (kStages + 1) * kNT * 4;        // row-id ring
    static constexpr int kTotal = kStages * kStage + kP + kHead + kRows;
};

// Tensor-core tile step (mma.sync m16n8k16, bf16 in, fp32 accumulate): the G
// query heads are the M rows of one 16-row fragment (rows >= G are zero).
//   logits  S[G x 64]  = Q[G x D] . K_tile^T   -- warp w: tile rows 16w .. 16w+15
//   output  O[G x D]  += P[G x 64] . V_tile    -- warp w: dims w*D/4 .. (w+1)*D/4-1
// P is rounded to bf16 for the product (the operand type of the tensor-core
// instruction); m, l and the rescaling stay fp32.
template <int D, int G>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const AttnArgs a) {
    using Lay = AttnLayout<D, G>;
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    constexpr int QCH = G * D * 2 / 16;        // 16-byte chunks of the queries
    constexpr int KST = D / 16;                // k-steps of the logit product
    constexpr int NTW = D / 32;                // 8-dim output tiles per warp

    extern __shared__ __align__(128) uint8_t smem[];
    float* ps = reinterpret_cast<float*>(smem + kStages * Lay::kStage);
    float* hm = ps + G * kPS;                  // running max per head (log2 domain)
    float* hl = hm + 16;                       // running sum per head
    float* ha = hl + 16;                       // rescale factor of the current tile
    int* rowbuf = reinterpret_cast<int*>(ha + 16);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;    // mma fragment coordinates
    const int p = blockIdx.x;
    const long long w0 = (long long)p * a.total_tiles / a.ctas;
    const long long w1 = (long long)(p + 1) * a.total_tiles / a.ctas;
    const int ntiles = (int)(w1 - w0);
    const size_t tstride = (size_t)a.hkv * Lay::kRowBytes;

    pdl_launch_dependents();
    pdl_wait();   // the index sets come from the previous kernel

    // index row j (< kNT) of local tile i, validated; -1 = no row
    auto fetch_row = [&](int i, int j) -> int {
        if (i >= ntiles) return -1;
        const int w = (int)(w0 + i);
        const int u = w / a.tiles_per_unit;
        const int e = (w - u * a.tiles_per_unit) * kNT + j;
        if (e >= a.B) return -1;
        int t = __ldcg(a.idx + (size_t)u * a.B + e);
        if (t < -1 || t >= a.T) {
            set_status(a.status, kStatusBadIndex);
            t = -1;
        }
        return t;
    };
    // row ids of local tile i live in rowbuf[i % (kStages + 1)] from the
    // iteration before it is issued until its compute is done
    auto rows_of = [&](int i) { return rowbuf + (i % (kStages + 1)) * kNT; };
    // all threads issue local tile i: 16 consecutive lanes copy one 256-byte
    // row (coalesced), then the unit's queries; one commit group per call
    auto issue = [&](int i) {
        if (i < ntiles) {
            uint8_t* st = smem + (i % kStages) * Lay::kStage;
            const int w = (int)(w0 + i);
            const int u = w / a.tiles_per_unit;
            const int b = u / a.hkv, h = u - b * a.hkv;
            const int* rows = rows_of(i);
            const uint8_t* kb = a.k + ((size_t)b * a.kv_bstride_rows + h) * Lay::kRowBytes;
            const uint8_t* vb = a.v + ((size_t)b * a.kv_bstride_rows + h) * Lay::kRowBytes;
#pragma unroll 4
            for (int id = tid; id < kNT * CPR; id += kAttnThreads) {
                const int j = id / CPR, c = id - j * CPR;
                const int t = rows[j];
                const size_t off = t >= 0 ? (size_t)t * tstride + c * 16 : 0;
                const uint32_t n = t >= 0 ? 16u : 0u;
                const int pc = swz(j, c);
                cp_async16(st + j * Lay::kRowBytes + pc * 16, kb + off, n);
                cp_async16(st + Lay::kKV + j * Lay::kRowBytes + pc * 16, vb + off, n);
            }
            const uint8_t* qs = reinterpret_cast<const uint8_t*>(a.q + ((size_t)b * a.hq + (size_t)h * G) * D);
            for (int c = tid; c < QCH; c += kAttnThreads) cp_async16(st + 2 * Lay::kKV + c * 16, qs + c * 16, 16u);
        }
        cp_async_commit();
    };

    // prologue: ids of the first kStages tiles (loads issued together), then
    // those tiles in flight, then the ids of the next tile in registers
    {
        int t0[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) t0[s] = tid < kNT ? fetch_row(s, tid) : -1;
        if (tid < kNT)
#pragma unroll
            for (int s = 0; s < kStages; ++s) rows_of(s)[tid] = t0[s];
        if (tid < 16) {
            hm[tid] = -INFINITY;
            hl[tid] = 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int s = 0; s < kStages; ++s) issue(s);
    }
    int t_next = tid < kNT ? fetch_row(kStages, tid) : -1;

    float acc[NTW][4];
#pragma unroll
    for (int j = 0; j < NTW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    __shared__ int s_last;

    for (int i = 0; i < ntiles; ++i) {
        const int s = i % kStages;
        if (tid < kNT) rows_of(i + kStages)[tid] = t_next;   // ids of the tile issued below
        cp_async_wait<kStages - 1>();
        __syncthreads();
        const uint8_t* ks = smem + s * Lay::kStage;
        const uint8_t* vs = ks + Lay::kKV;
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(ks + 2 * Lay::kKV);
        const int* rows = rows_of(i);
        const int w = (int)(w0 + i);
        const int u = w / a.tiles_per_unit;

        // ---- logits for tile rows 16w .. 16w+15 (two 8-row n-tiles)
        {
            float sacc[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
            const int mi = lane >> 3, r8 = lane & 7;
            const int krow = (warp * 2 + (mi >> 1)) * 8 + r8;
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                uint32_t af[4];
                af[0] = g < G ? qw[(g * D + kk * 16 + 2 * t4) >> 1] : 0u;
                af[1] = g + 8 < G ? qw[((g + 8) * D + kk * 16 + 2 * t4) >> 1] : 0u;
                af[2] = g < G ? qw[(g * D + kk * 16 + 8 + 2 * t4) >> 1] : 0u;
                af[3] = g + 8 < G ? qw[((g + 8) * D + kk * 16 + 8 + 2 * t4) >> 1] : 0u;
                uint32_t bf[4];
                ldsm_x4(bf, ks + krow * Lay::kRowBytes + swz(krow, kk * 2 + (mi & 1)) * 16);
                mma_bf16(sacc[0], af, bf[0], bf[1]);
                mma_bf16(sacc[1], af, bf[2], bf[3]);
            }
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int r0 = (warp * 2 + n) * 8 + 2 * t4;
                const bool v0 = rows[r0] >= 0, v1 = rows[r0 + 1] >= 0;
                if (g < G) {
                    ps[g * kPS + r0] = v0 ? sacc[n][0] * a.qscale : -INFINITY;
                    ps[g * kPS + r0 + 1] = v1 ? sacc[n][1] * a.qscale : -INFINITY;
                }
                if (g + 8 < G) {
                    ps[(g + 8) * kPS + r0] = v0 ? sacc[n][2] * a.qscale : -INFINITY;
                    ps[(g + 8) * kPS + r0 + 1] = v1 ? sacc[n][3] * a.qscale : -INFINITY;
                }
            }
        }
        __syncthreads();

        // ---- online softmax per head (warp w: heads w, w + 4, ...)
        for (int hh = warp; hh < G; hh += kAttnWarps) {
            float* pg = ps + hh * kPS;
            const float x0 = pg[lane], x1 = pg[lane + 32];
            const float tmax = warp_max(fmaxf(x0, x1));
            const float m_old = hm[hh];
            const float m_new = fmaxf(m_old, tmax);
            float e0 = 0.f, e1 = 0.f, alpha = 1.f;
            if (m_new != -INFINITY) {
                alpha = exp2f(m_old - m_new);
                e0 = exp2f(x0 - m_new);
                e1 = exp2f(x1 - m_new);
            }
            pg[lane] = e0;
            pg[lane + 32] = e1;
            const float lsum = warp_sum(e0 + e1);
            if (lane == 0) {
                hl[hh] = hl[hh] * alpha + lsum;
                hm[hh] = m_new;
                ha[hh] = alpha;
            }
        }
        __syncthreads();

        // ---- rescale and accumulate P . V for this warp's dims
        {
            const float al0 = g < G ? ha[g] : 1.f, al1 = g + 8 < G ? ha[g + 8] : 1.f;
#pragma unroll
            for (int j = 0; j < NTW; ++j) {
                acc[j][0] *= al0;
                acc[j][1] *= al0;
                acc[j][2] *= al1;
                acc[j][3] *= al1;
            }
            const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
            for (int kq = 0; kq < kNT / 16; ++kq) {
                uint32_t af[4];
                const int c0 = kq * 16 + 2 * t4;
                af[0] = g < G ? pack_bf16(ps[g * kPS + c0], ps[g * kPS + c0 + 1]) : 0u;
                af[1] = g + 8 < G ? pack_bf16(ps[(g + 8) * kPS + c0], ps[(g + 8) * kPS + c0 + 1]) : 0u;
                af[2] = g < G ? pack_bf16(ps[g * kPS + c0 + 8], ps[g * kPS + c0 + 9]) : 0u;
                af[3] = g + 8 < G ? pack_bf16(ps[(g + 8) * kPS + c0 + 8], ps[(g + 8) * kPS + c0 + 9]) : 0u;
                const int vrow = kq * 16 + (mi & 1) * 8 + r8;
#pragma unroll
                for (int j = 0; j < NTW; j += 2) {
                    const int nt = warp * NTW + j + (mi >> 1);
                    uint32_t bf[4];
                    ldsm_x4_t(bf, vs + vrow * Lay::kRowBytes + swz(vrow, nt) * 16);
                    mma_bf16(acc[j], af, bf[0], bf[1]);
                    mma_bf16(acc[j + 1], af, bf[2], bf[3]);
                }
            }
        }
        __syncthreads();   // stage s and the logits are free again

        // refill stage s with tile i + kStages; fetch the ids one tile further
        issue(i + kStages);
        t_next = tid < kNT ? fetch_row(i + kStages + 1, tid) : -1;

        // ---- end of a segment: this CTA's last tile of unit u
        const bool seg_end = i + 1 == ntiles || (w + 1) / a.tiles_per_unit != u;
        if (!seg_end) continue;
        const int b = u / a.hkv, h = u - b * a.hkv;
        const long long wu0 = (long long)u * a.tiles_per_unit;
        const int pfirst = owner(wu0, a);
        const int nslot = owner(wu0 + a.tiles_per_unit - 1, a) - pfirst + 1;
        if (nslot == 1) {
            // the whole unit lies in this CTA: write the output directly
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int hd = g + 8 * half;
                if (hd < G) {
                    const float l = hl[hd];
                    const float inv = l > 0.f ? 1.f / l : 0.f;
                    uint16_t* o = a.out + ((size_t)b * a.hq + h * G + hd) * D;
#pragma unroll
                    for (int j = 0; j < NTW; ++j) {
                        const int d0 = (warp * NTW + j) * 8 + 2 * t4;
                        *reinterpret_cast<uint32_t*>(o + d0) =
                            pack_bf16(acc[j][2 * half] * inv, acc[j][2 * half + 1] * inv);
                    }
                }
            }
        } else {
            const int slot = p - pfirst;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int hd = g + 8 * half;
                if (hd < G) {
                    const size_t pi = ((size_t)u * a.smax + slot) * G + hd;
                    if (warp == 0 && t4 == 0) {
                        a.pm[pi] = hm[hd];
                        a.pl[pi] = hl[hd];
                    }
                    float* po = a.po + pi * D;
#pragma unroll
                    for (int j = 0; j < NTW; ++j) {
                        const int d0 = (warp * NTW + j) * 8 + 2 * t4;
                        *reinterpret_cast<float2*>(po + d0) = make_float2(acc[j][2 * half], acc[j][2 * half + 1]);
                    }
                }
            }
            __syncthreads();
            if (tid == 0) {
                unsigned old;
                asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + u) : "memory");
                s_last = old + 1 == (unsigned)nslot;
                if (s_last) a.counters[u] = 0u;
            }
            __syncthreads();
            if (s_last) {
                __threadfence();
                // merge the unit's nslot partials: warp -> heads, lanes -> slots for
                // the weights, then lanes -> dims with every slot's loads in flight
                constexpr int DPL = D / 32;
                for (int hd = warp; hd < G; hd += kAttnWarps) {
                    const size_t base = (size_t)u * a.smax * G + hd;
                    float M = -INFINITY;
                    for (int x = lane; x < nslot; x += 32) M = fmaxf(M, __ldcg(a.pm + base + (size_t)x * G));
                    M = warp_max(M);
                    float L = 0.f, oacc[DPL];
#pragma unroll
                    for (int k = 0; k < DPL; ++k) oacc[k] = 0.f;
                    if (M != -INFINITY) {
                        for (int x0 = 0; x0 < nslot; x0 += 8) {
                            float wv[8], vals[8][DPL];
#pragma unroll
                            for (int y = 0; y < 8; ++y) {
                                const int x = x0 + y;
                                const size_t pi = base + (size_t)x * G;
                                const float mx = x < nslot ? __ldcg(a.pm + pi) : -INFINITY;
                                wv[y] = mx == -INFINITY ? 0.f : exp2f(mx - M);
                                const float lx = x < nslot ? __ldcg(a.pl + pi) : 0.f;
                                L = fmaf(wv[y], lx, L);
#pragma unroll
                                for (int k = 0; k < DPL; ++k)
                                    vals[y][k] = x < nslot ? __ldcg(a.po + pi * D + lane * DPL + k) : 0.f;
                            }
#pragma unroll
                            for (int y = 0; y < 8; ++y)
#pragma unroll
                                for (int k = 0; k < DPL; ++k) oacc[k] = fmaf(wv[y], vals[y][k], oacc[k]);
                        }
                    }
                    const float inv = L > 0.f ? 1.f / L : 0.f;
                    uint16_t* o = a.out + ((size_t)b * a.hq + h * G + hd) * D + lane * DPL;
#pragma unroll
                    for (int k = 0; k < DPL; ++k) o[k] = f2bf(oacc[k] * inv);
                }
            }
        }
        // next segment: fresh state (the barrier at the top of the next
        // iteration orders these resets before their first use)
#pragma unroll
        for (int j = 0; j < NTW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        __syncthreads();
        if (tid < 16) {
            hm[tid] = -INFINITY;
            hl[tid] = 0.f;
        }
    }
    cp_async_wait<0>();
}

template <int D, int G>
cudaError_t launch_attn_t(const LaunchCtx& ctx, AttnArgs a) {
    using Lay = AttnLayout<D, G>;
    const size_t smem = Lay::kTotal;
    auto kern = attn_kernel<D, G>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)a.ctas);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_attn_d(const LaunchCtx& ctx, const AttnArgs& a, int G) {
    switch (G) {
        case 1: return launch_attn_t<D, 1>(ctx, a);
        case 2: return launch_attn_t<D, 2>(ctx, a);
        case 4: return launch_attn_t<D, 4>(ctx, a);
        case 8: return launch_attn_t<D, 8>(ctx, a);
        case 16: return launch_attn_t<D, 16>(ctx, a);
        default: return cudaErrorInvalidValue;
    }
}

template <int D>
size_t smem_d(int G) {
    switch (G) {
        case 1: return AttnLayout<D, 1>::kTotal;
        case 2: return AttnLayout<D, 2>::kTotal;
        case 4: return AttnLayout<D, 4>::kTotal;
        case 8: return AttnLayout<D, 8>::kTotal;
        default: return AttnLayout<D, 16>::kTotal;
    }
}

}  // namespace

AttnPlan plan_attn(int nb, int hkv, int G, int B, int d, int num_sms) {
    AttnPlan p{};
    p.units = (long long)nb * hkv;
    p.tiles_per_unit = (B + kNT - 1) / kNT;
    p.total_tiles = p.units * p.tiles_per_unit;
    const size_t smem = d == 64 ? smem_d<64>(G) : (d == 128 ? smem_d<128>(G) : smem_d<256>(G));
    int per_sm = (int)(227 * 1024 / (smem + 1024));
    if (per_sm > 4) per_sm = 4;
    if (per_sm < 1) per_sm = 1;
    long long ctas = (long long)num_sms * per_sm;
    if (ctas > p.total_tiles) ctas = p.total_tiles;
    p.ctas = (int)ctas;
    const long long per = p.total_tiles / ctas;   // >= 1
    long long smax = (p.tiles_per_unit - 1) / per + 2;
    if (smax > p.tiles_per_unit) smax = p.tiles_per_unit;
    p.smax = (int)smax;
    return p;
}

cudaError_t launch_attn(const LaunchCtx& ctx, const AttnPlan& plan, const uint16_t* q, const uint16_t* k,
                        const uint16_t* v, const int32_t* idx, int B, float scale, uint16_t* out, float* pm, float* pl,
                        float* po, unsigned* counters, int nb, int hq, int hkv, int d, int T,
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
    a.counters = counters;
    a.kv_bstride_rows = kv_bstride_rows;
    a.hq = hq;
    a.hkv = hkv;
    a.T = T;
    a.B = B;
    a.units = (int)plan.units;
    a.tiles_per_unit = plan.tiles_per_unit;
    a.ctas = plan.ctas;
    a.smax = plan.smax;
    a.total_tiles = plan.total_tiles;
    a.qscale = scale * kLog2e;
    a.status = status;
    (void)nb;
    const int G = hq / hkv;
    switch (d) {
        case 64: return launch_attn_d<64>(ctx, a, G);
        case 128: return launch_attn_d<128>(ctx, a, G);
        case 256: return launch_attn_d<256>(ctx, a, G);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
