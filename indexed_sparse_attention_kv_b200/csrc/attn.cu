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
// ranges, one per CTA (P = one wave). A CTA streams its tiles through a
// kStages-deep ring: the selected K and V rows land in shared memory by 16-byte
// cp.async, 16 consecutive lanes per 256-byte row (coalesced), in an XOR
// swizzle that keeps every ldmatrix phase conflict-free; padded entries are
// zero-filled. The row ids of the tile kStages ahead are read one iteration
// early. (Per-row TMA bulk copies were measured slower for 256-byte rows: the
// copy engine, not DRAM, became the limit.)
//
// Compute (tensor cores, mma.sync m16n8k16, bf16 in, fp32 accumulate): the G
// query heads are the M rows of one 16-row fragment (rows >= G are zero), and
// warp w owns rows 16w .. 16w+15 of every tile, FlashAttention-2 style: it
// forms its 16 logits per head, keeps a running max / sum per head in
// registers, turns the probabilities (rounded to bf16, the operand type of the
// instruction) straight from the logit fragments into the A operand of P.V,
// and accumulates O[G x d] in registers. The 4 warps' states are merged through
// shared memory at the end of a segment (the CTA's part of one unit). A unit
// contained in one CTA is written directly; otherwise the CTA writes a partial
// and the last one to finish a unit (a release/acquire counter, left at zero)
// merges the unit's partials.
//
// Cluster mode (few units, as in batched decode): when every unit can own a
// cluster of C CTAs (16, else 8) in one wave and has C to 4 * C (C = 16) or
// 8 * C (C = 8) tiles, CTA r of unit u's cluster takes tiles r * n / C ..
// (r + 1) * n / C - 1 of the unit, and the cluster merges its partials through
// distributed shared memory (each CTA produces 1 / C of the unit's outputs),
// with no global partials, counters or second pass over L2.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {

namespace {

namespace cg = cooperative_groups;

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = 4;
constexpr int kNT = 64;               // index-set entries per tile (16 per warp)
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
    long long kv_bstride_rows;   // T * hkv for decode, 0 for prefill (one shared cache) and paged pools
    const int32_t* slots;        // optional page table (page size 1): [nb, T] pool row of position t
    long long nslots;            // rows of the K/V pools when paged
    int hq, hkv, T, B;
    int units, tiles_per_unit, ctas, smax;
    long long total_tiles;
    float qscale;             // scale * log2(e)
    unsigned* status;
    long long wait_limit;
};

// CTA that owns flattened tile w (ranges lo_p = p * W / P).
__device__ __forceinline__ int owner(long long w, const AttnArgs& a) {
    return (int)(((w + 1) * (long long)a.ctas - 1) / a.total_tiles);
}

// Swizzled position of 16-byte chunk c of tile row j: the 8 rows of an
// ldmatrix phase hit 8 distinct 16-byte bank groups.
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
__device__ __forceinline__ float quad_max(float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

template <int D, int G>
struct AttnLayout {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kKV = kNT * kRowBytes;                    // one of K or V per stage
    static constexpr int kQ = G * D * 2;                           // the unit's queries (bf16)
    static constexpr int kStage = (2 * kKV + kQ + 127) / 128 * 128;
    static constexpr int kMerge = (kAttnWarps - 1) * (G * D + 2 * 16) * 4;   // warps 1..3: O, m, l
    static constexpr int kRows = 4 * kNT * 4;                      // row-id ring (>= stages + 1)
    static constexpr int kFixed = kMerge + kRows;
    // two stages: three CTAs (12 warps) fit per SM, which hides the fixed
    // latencies of the per-warp MMA / softmax chain better than a third stage
    static constexpr int kStages = 2;
    static constexpr int kTotal = kStages * kStage + kFixed;
};

template <int D, int G, bool PAGED, int CL>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const AttnArgs a) {
    using Lay = AttnLayout<D, G>;
    constexpr int S = Lay::kStages;
    constexpr int KST = D / 16;                // k-steps of the logit product
    constexpr int NTO = D / 8;                 // 8-dim output tiles
    static_assert(S + 1 <= 4, "row-id ring");

    extern __shared__ __align__(128) uint8_t smem[];
    float* merge = reinterpret_cast<float*>(smem + S * Lay::kStage);
    int* rowbuf = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(merge) + Lay::kMerge);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;    // mma fragment coordinates
    const int p = blockIdx.x;
    // stream-K: contiguous ranges of the flattened tiles; cluster mode: CTA r
    // of cluster u takes its share of unit u's tiles (at least one)
    const long long w0 = CL ? (long long)(p / CL) * a.tiles_per_unit + (long long)(p % CL) * a.tiles_per_unit / CL
                            : (long long)p * a.total_tiles / a.ctas;
    const long long w1 = CL ? (long long)(p / CL) * a.tiles_per_unit + (long long)(p % CL + 1) * a.tiles_per_unit / CL
                            : (long long)(p + 1) * a.total_tiles / a.ctas;
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
        if (PAGED && t >= 0) {   // logical position -> pool row
            const int p = __ldg(a.slots + (size_t)(u / a.hkv) * a.T + t);
            if (p < 0 || p >= a.nslots) {
                set_status(a.status, kStatusBadIndex);
                t = -1;
            } else {
                t = p;
            }
        }
        return t;
    };
    auto rows_of = [&](int i) { return rowbuf + (i & 3) * kNT; };
    // all threads issue local tile i: 16 consecutive lanes copy one 256-byte
    // row (coalesced), then the unit's queries; one commit group per call
    auto issue = [&](int i) {
        if (i < ntiles) {
            uint8_t* st = smem + (i % S) * Lay::kStage;
            const int w = (int)(w0 + i);
            const int u = w / a.tiles_per_unit;
            const int b = u / a.hkv, h = u - b * a.hkv;
            const int* rows = rows_of(i);
            const uint8_t* kb = a.k + ((size_t)b * a.kv_bstride_rows + h) * Lay::kRowBytes;
            const uint8_t* vb = a.v + ((size_t)b * a.kv_bstride_rows + h) * Lay::kRowBytes;
            constexpr int CPR = D / 8;
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
            for (int c = tid; c < Lay::kQ / 16; c += kAttnThreads) cp_async16(st + 2 * Lay::kKV + c * 16, qs + c * 16, 16u);
        }
        cp_async_commit();
    };

    // prologue: ids of the first S tiles (loads issued together), then those
    // tiles in flight, then the ids of the next tile in registers
    {
        int t0[S];
#pragma unroll
        for (int s = 0; s < S; ++s) t0[s] = tid < kNT ? fetch_row(s, tid) : -1;
        if (tid < kNT)
#pragma unroll
            for (int s = 0; s < S; ++s) rows_of(s)[tid] = t0[s];
        __syncthreads();   // ids visible
#pragma unroll
        for (int s = 0; s < S; ++s) issue(s);
    }
    int t_next = tid < kNT ? fetch_row(S, tid) : -1;

    // per-warp running state: heads g (c0/c1 rows) and g + 8 (c2/c3 rows)
    float acc[NTO][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint32_t qf[KST][4];
    int cur_u = -1;
    __shared__ int s_last;
#pragma unroll
    for (int j = 0; j < NTO; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    for (int i = 0; i < ntiles; ++i) {
        const int s = i % S;
        if (tid < kNT) rows_of(i + S)[tid] = t_next;   // ids of the tile issued below
        cp_async_wait<S - 1>();
        __syncthreads();   // tile i visible to every thread
        const uint8_t* ks = smem + s * Lay::kStage;
        const uint8_t* vs = ks + Lay::kKV;
        const int* rows = rows_of(i);
        const int w = (int)(w0 + i);
        const int u = w / a.tiles_per_unit;
        if (u != cur_u) {   // a new unit: its query fragments (A operand, rows >= G zero)
            cur_u = u;
            const uint32_t* qw = reinterpret_cast<const uint32_t*>(ks + 2 * Lay::kKV);
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                qf[kk][0] = g < G ? qw[(g * D + kk * 16 + 2 * t4) >> 1] : 0u;
                qf[kk][1] = g + 8 < G ? qw[((g + 8) * D + kk * 16 + 2 * t4) >> 1] : 0u;
                qf[kk][2] = g < G ? qw[(g * D + kk * 16 + 8 + 2 * t4) >> 1] : 0u;
                qf[kk][3] = g + 8 < G ? qw[((g + 8) * D + kk * 16 + 8 + 2 * t4) >> 1] : 0u;
            }
        }

        // ---- logits of this warp's 16 tile rows (two 8-row n-tiles)
        float sc[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
        {
            const int mi = lane >> 3, r8 = lane & 7;
            const int krow = warp * 16 + (mi >> 1) * 8 + r8;
            const uint8_t* kp = ks + krow * Lay::kRowBytes;
#pragma unroll
            for (int kk = 0; kk < KST; ++kk) {
                uint32_t bf[4];
                ldsm_x4(bf, kp + swz(krow, kk * 2 + (mi & 1)) * 16);
                mma_bf16(sc[0], qf[kk], bf[0], bf[1]);
                mma_bf16(sc[1], qf[kk], bf[2], bf[3]);
            }
        }
        // ---- online softmax per head row (the 4 lanes of a quad hold one row)
        float pr[2][4];
        {
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int r0 = warp * 16 + n * 8 + 2 * t4;
                const bool v0 = rows[r0] >= 0, v1 = rows[r0 + 1] >= 0;
                sc[n][0] = v0 ? sc[n][0] * a.qscale : -INFINITY;
                sc[n][1] = v1 ? sc[n][1] * a.qscale : -INFINITY;
                sc[n][2] = v0 ? sc[n][2] * a.qscale : -INFINITY;
                sc[n][3] = v1 ? sc[n][3] * a.qscale : -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
            }
            mx0 = quad_max(mx0);
            mx1 = quad_max(mx1);
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
            const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                pr[n][0] = mn0 == -INFINITY ? 0.f : exp2f(sc[n][0] - mn0);
                pr[n][1] = mn0 == -INFINITY ? 0.f : exp2f(sc[n][1] - mn0);
                pr[n][2] = mn1 == -INFINITY ? 0.f : exp2f(sc[n][2] - mn1);
                pr[n][3] = mn1 == -INFINITY ? 0.f : exp2f(sc[n][3] - mn1);
                s0 += pr[n][0] + pr[n][1];
                s1 += pr[n][2] + pr[n][3];
            }
            l0 = l0 * al0 + quad_sum(s0);
            l1 = l1 * al1 + quad_sum(s1);
            m0 = mn0;
            m1 = mn1;
#pragma unroll
            for (int j = 0; j < NTO; ++j) {
                acc[j][0] *= al0;
                acc[j][1] *= al0;
                acc[j][2] *= al1;
                acc[j][3] *= al1;
            }
        }
        // ---- O += P . V over this warp's 16 rows (one k-step)
        {
            uint32_t af[4];
            af[0] = pack_bf16(pr[0][0], pr[0][1]);
            af[1] = pack_bf16(pr[0][2], pr[0][3]);
            af[2] = pack_bf16(pr[1][0], pr[1][1]);
            af[3] = pack_bf16(pr[1][2], pr[1][3]);
            const int mi = lane >> 3, r8 = lane & 7;
            const int vrow = warp * 16 + (mi & 1) * 8 + r8;
            const uint8_t* vp = vs + vrow * Lay::kRowBytes;
#pragma unroll
            for (int j = 0; j < NTO; j += 2) {
                uint32_t bf[4];
                ldsm_x4_t(bf, vp + swz(vrow, j + (mi >> 1)) * 16);
                mma_bf16(acc[j], af, bf[0], bf[1]);
                mma_bf16(acc[j + 1], af, bf[2], bf[3]);
            }
        }

        __syncthreads();   // stage s free once every warp is done with it
        issue(i + S);
        t_next = tid < kNT ? fetch_row(i + S + 1, tid) : -1;

        // ---- end of a segment: this CTA's last tile of unit u
        const bool seg_end = i + 1 == ntiles || (w + 1) / a.tiles_per_unit != u;
        if (!seg_end) continue;
        // merge the 4 warps' states into warp 0 (rows g and g + 8 of each)
        if (warp > 0) {
            float* mw = merge + (warp - 1) * (G * D + 32);
            if (t4 == 0) {
                mw[G * D + g] = m0;
                mw[G * D + 16 + g] = l0;
                if (g + 8 < 16) {
                    mw[G * D + g + 8] = m1;
                    mw[G * D + 16 + g + 8] = l1;
                }
            }
#pragma unroll
            for (int j = 0; j < NTO; ++j) {
                const int d0 = j * 8 + 2 * t4;
                if (g < G) *reinterpret_cast<float2*>(mw + g * D + d0) = make_float2(acc[j][0], acc[j][1]);
                if (g + 8 < G) *reinterpret_cast<float2*>(mw + (g + 8) * D + d0) = make_float2(acc[j][2], acc[j][3]);
            }
        }
        __syncthreads();
        const int b = u / a.hkv, h = u - b * a.hkv;
        const long long wu0 = (long long)u * a.tiles_per_unit;
        const int pfirst = CL ? 0 : owner(wu0, a);
        const int nslot = CL ? CL : owner(wu0 + a.tiles_per_unit - 1, a) - pfirst + 1;
        if (warp == 0) {
            float M0 = m0, M1 = m1;
#pragma unroll
            for (int x = 0; x < kAttnWarps - 1; ++x) {
                const float* mw = merge + x * (G * D + 32);
                M0 = fmaxf(M0, mw[G * D + g]);
                M1 = fmaxf(M1, g + 8 < 16 ? mw[G * D + g + 8] : -INFINITY);
            }
            float w00 = M0 == -INFINITY ? 0.f : exp2f(m0 - M0), w10 = M1 == -INFINITY ? 0.f : exp2f(m1 - M1);
            float L0 = w00 * l0, L1 = w10 * l1;
#pragma unroll
            for (int j = 0; j < NTO; ++j) {
                acc[j][0] *= w00;
                acc[j][1] *= w00;
                acc[j][2] *= w10;
                acc[j][3] *= w10;
            }
#pragma unroll
            for (int x = 0; x < kAttnWarps - 1; ++x) {
                const float* mw = merge + x * (G * D + 32);
                const float wx0 = M0 == -INFINITY ? 0.f : exp2f(mw[G * D + g] - M0);
                const float wx1 = M1 == -INFINITY ? 0.f : exp2f(mw[G * D + g + 8] - M1);
                L0 = fmaf(wx0, mw[G * D + 16 + g], L0);
                L1 = fmaf(wx1, mw[G * D + 16 + g + 8], L1);
#pragma unroll
                for (int j = 0; j < NTO; ++j) {
                    const int d0 = j * 8 + 2 * t4;
                    if (g < G) {
                        const float2 o = *reinterpret_cast<const float2*>(mw + g * D + d0);
                        acc[j][0] = fmaf(wx0, o.x, acc[j][0]);
                        acc[j][1] = fmaf(wx0, o.y, acc[j][1]);
                    }
                    if (g + 8 < G) {
                        const float2 o = *reinterpret_cast<const float2*>(mw + (g + 8) * D + d0);
                        acc[j][2] = fmaf(wx1, o.x, acc[j][2]);
                        acc[j][3] = fmaf(wx1, o.y, acc[j][3]);
                    }
                }
            }
            if constexpr (CL > 0) {
                // this CTA's partial for the cluster: the stage ring is idle (the
                // unit's last tile is consumed and nothing is in flight)
                float* cp = reinterpret_cast<float*>(smem);
                if (t4 == 0) {
                    if (g < G) {
                        cp[g] = M0;
                        cp[16 + g] = L0;
                    }
                    if (g + 8 < G) {
                        cp[g + 8] = M1;
                        cp[16 + g + 8] = L1;
                    }
                }
#pragma unroll
                for (int j = 0; j < NTO; ++j) {
                    const int d0 = j * 8 + 2 * t4;
                    if (g < G) *reinterpret_cast<float2*>(cp + 32 + g * D + d0) = make_float2(acc[j][0], acc[j][1]);
                    if (g + 8 < G)
                        *reinterpret_cast<float2*>(cp + 32 + (g + 8) * D + d0) = make_float2(acc[j][2], acc[j][3]);
                }
            } else if (nslot == 1) {
                // the whole unit lies in this CTA: write the output directly
                const float i0 = L0 > 0.f ? 1.f / L0 : 0.f, i1 = L1 > 0.f ? 1.f / L1 : 0.f;
#pragma unroll
                for (int j = 0; j < NTO; ++j) {
                    const int d0 = j * 8 + 2 * t4;
                    if (g < G)
                        *reinterpret_cast<uint32_t*>(a.out + ((size_t)b * a.hq + h * G + g) * D + d0) =
                            pack_bf16(acc[j][0] * i0, acc[j][1] * i0);
                    if (g + 8 < G)
                        *reinterpret_cast<uint32_t*>(a.out + ((size_t)b * a.hq + h * G + g + 8) * D + d0) =
                            pack_bf16(acc[j][2] * i1, acc[j][3] * i1);
                }
            } else {
                const int slot = p - pfirst;
                const size_t pi0 = ((size_t)u * a.smax + slot) * G + g;
                if (t4 == 0) {
                    if (g < G) {
                        a.pm[pi0] = M0;
                        a.pl[pi0] = L0;
                    }
                    if (g + 8 < G) {
                        a.pm[pi0 + 8] = M1;
                        a.pl[pi0 + 8] = L1;
                    }
                }
#pragma unroll
                for (int j = 0; j < NTO; ++j) {
                    const int d0 = j * 8 + 2 * t4;
                    if (g < G) *reinterpret_cast<float2*>(a.po + pi0 * D + d0) = make_float2(acc[j][0], acc[j][1]);
                    if (g + 8 < G)
                        *reinterpret_cast<float2*>(a.po + (pi0 + 8) * D + d0) = make_float2(acc[j][2], acc[j][3]);
                }
            }
        }
        if constexpr (CL > 0) {
            // every CTA of the cluster reaches this point once (its last tile
            // ends its only segment); merge slice r of the unit's G x D outputs
            // from the CL partials in the cluster's shared memory
            cg::cluster_group cluster = cg::this_cluster();
            cluster.sync();
            const float* parts[CL];
#pragma unroll
            for (int c = 0; c < CL; ++c) parts[c] = cluster.map_shared_rank(reinterpret_cast<const float*>(smem), c);
            const int r = (int)cluster.block_rank();
            const int e0 = r * (G * D) / CL, e1 = (r + 1) * (G * D) / CL;
            for (int e = e0 + tid; e < e1; e += kAttnThreads) {
                const int hd = e / D;
                float mc[CL];
                float M = -INFINITY;
#pragma unroll
                for (int c = 0; c < CL; ++c) {
                    mc[c] = parts[c][hd];
                    M = fmaxf(M, mc[c]);
                }
                float L = 0.f, O = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int c = 0; c < CL; ++c) {
                        const float wc = exp2f(mc[c] - M);
                        L = fmaf(wc, parts[c][16 + hd], L);
                        O = fmaf(wc, parts[c][32 + e], O);
                    }
                }
                const float inv = L > 0.f ? 1.f / L : 0.f;
                a.out[((size_t)b * a.hq + h * G) * D + e] = f2bf(O * inv);
            }
            cluster.sync();   // keep this CTA's partial alive for remote readers
        } else if (nslot > 1) {
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
                // merge the unit's nslot partials: warp -> heads; lanes -> slots for
                // the weights, then lanes -> dims with 16 slots' loads in flight
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
                        for (int x0 = 0; x0 < nslot; x0 += 32) {
                            const int xl = x0 + lane;
                            const float mx = xl < nslot ? __ldcg(a.pm + base + (size_t)xl * G) : -INFINITY;
                            const float lx = xl < nslot ? __ldcg(a.pl + base + (size_t)xl * G) : 0.f;
                            const float wl = mx == -INFINITY ? 0.f : exp2f(mx - M);
                            L += warp_sum(wl * lx);
                            const int cnt = min(32, nslot - x0);
                            for (int y0 = 0; y0 < cnt; y0 += 16) {
                                float vals[16][DPL];
#pragma unroll
                                for (int y = 0; y < 16; ++y)
#pragma unroll
                                    for (int k = 0; k < DPL; ++k)
                                        vals[y][k] = y0 + y < cnt
                                                         ? __ldcg(a.po + (base + (size_t)(x0 + y0 + y) * G) * D + lane * DPL + k)
                                                         : 0.f;
#pragma unroll
                                for (int y = 0; y < 16; ++y) {
                                    const float wy = __shfl_sync(0xffffffffu, wl, (y0 + y) & 31);
#pragma unroll
                                    for (int k = 0; k < DPL; ++k) oacc[k] = fmaf(wy, vals[y][k], oacc[k]);
                                }
                            }
                        }
                    }
                    const float inv = L > 0.f ? 1.f / L : 0.f;
                    uint16_t* o = a.out + ((size_t)b * a.hq + h * G + hd) * D + lane * DPL;
#pragma unroll
                    for (int k = 0; k < DPL; ++k) o[k] = f2bf(oacc[k] * inv);
                }
            }
        }
        // next segment: fresh state (the merge buffer is reused only after the
        // next segment end's barrier)
#pragma unroll
        for (int j = 0; j < NTO; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
        __syncthreads();
    }
    cp_async_wait<0>();
}

// Launches cluster mode with CL-CTA clusters if every unit has CL .. 8 * CL
// tiles (CL .. 4 * CL for 16-CTA clusters: a few per CTA, the latency-bound
// regime; with more, stream-K's fuller grid streams as fast or faster,
// measured over batch 1-8 and B 512-8192 at 128K) and all units' clusters are
// resident at once; *done tells whether it launched.
template <int D, int G, int CL>
cudaError_t try_cluster(const LaunchCtx& ctx, const AttnArgs& a, bool* done) {
    *done = false;
    const int max_per_cta = CL > 8 ? 4 : 8;
    if (a.tiles_per_unit < CL || a.tiles_per_unit > max_per_cta * CL || (long long)a.units * CL > 4ll * ctx.num_sms)
        return cudaSuccess;
    const size_t smem = AttnLayout<D, G>::kTotal;
    auto kern = a.slots ? attn_kernel<D, G, true, CL> : attn_kernel<D, G, false, CL>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    if (CL > 8) {   // beyond the portable cluster size
        static std::mutex mu;
        static std::map<std::pair<const void*, int>, bool> allowed;
        std::lock_guard<std::mutex> g(mu);
        bool& ok = allowed[{(const void*)kern, current_device()}];
        if (!ok) {
            if (cudaFuncSetAttribute((const void*)kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
                (void)cudaGetLastError();   // not offered: the caller tries the portable size
                return cudaSuccess;
            }
            ok = true;
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(a.units * CL));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    // without programmatic dependent launch: clusters placed while the
    // previous kernel's CTAs drain land on fragmented GPCs (128K decode
    // attention 15.0 us with PDL, 14.0 us without, measured)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cached_active_clusters((const void*)kern, cfg, &clusters) != cudaSuccess) {
        (void)cudaGetLastError();   // no answer: the caller falls back to a smaller cluster or stream-K
        return cudaSuccess;
    }
    if (clusters < a.units) return cudaSuccess;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    *done = true;
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_attn_t(const LaunchCtx& ctx, AttnArgs a) {
    // cluster mode: 16-CTA clusters (two tiles or more per CTA) when they all
    // fit, else 8-CTA clusters; otherwise stream-K
    bool done = false;
    cudaError_t e = try_cluster<D, G, 16>(ctx, a, &done);
    if (e != cudaSuccess || done) return e;
    e = try_cluster<D, G, 8>(ctx, a, &done);
    if (e != cudaSuccess || done) return e;
    const size_t smem = AttnLayout<D, G>::kTotal;
    auto kern = a.slots ? attn_kernel<D, G, true, 0> : attn_kernel<D, G, false, 0>;
    e = ensure_dyn_smem((const void*)kern, (int)smem);
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
    int per_sm = (int)(228 * 1024 / (smem + 1024));
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
                        long long kv_bstride_rows, unsigned* status, const int32_t* slots, long long nslots) {
    AttnArgs a{};
    a.slots = slots;
    a.nslots = nslots;
    if (slots) kv_bstride_rows = 0;
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
    a.wait_limit = ctx.wait_limit;
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
