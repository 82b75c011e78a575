// Prefill indexer: for every query row p of a prefill and every KV head h,
// the top-B positions t <= p of s[p,h,t] = q_bar[p,h] . kt[t,h] (LongCat
// Sparse Attention, Abstract: the Lightning Indexer's dense O(L^2) scoring;
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Fig. 1
// for the group-mean query).
//
// The scores are never materialised. The score GEMM runs on the tensor cores
// (tcgen05.mma, operands staged by TMA in 128-byte-swizzled shared memory,
// fp32 accumulators in TMEM), twice:
//   1. sample pass: only every S-th key column. A per-row radix select over
//      those samples gives a threshold theta_row that about 1.5 B of the
//      row's keys exceed (a row left with fewer than B is re-selected, below);
//   2. filter pass: all causal columns; the epilogue appends (score, position)
//      of every score >= theta_row to a per-row candidate list.
// A final per-row selection takes the exact top B of the candidates (ties:
// lower position) and writes them in ascending order through a position
// bitmap. Rows whose list overflowed its capacity or holds fewer than B keys
// (a sample that misjudged the row) are re-done exactly from scratch by the
// same kernel, recomputing scores on the CUDA cores.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "block_select.cuh"
#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {
namespace {

constexpr int kBM = 128;              // query rows per tile = TMEM lanes
constexpr int kBN = 256;              // key columns per tile = fp32 TMEM columns
constexpr int kGemmThreads = 384;     // warp 0 TMA, warp 1 MMA + TMEM owner, warps 4..11 epilogue
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 8;
constexpr int kAccCols = 2 * kBN;     // two accumulators (double-buffered)
constexpr int kMaxStages = 6;
constexpr int kSelThreads = 512;
constexpr int kMaxSamples = 8192;
constexpr int kMaxSlots = 8;
constexpr int kStageRow = 36;         // staging row pitch (floats): conflict-free 16-byte stores
constexpr int kStageFloats = 32 * kStageRow;          // writer slots per row (2 x at most 4 segments)
constexpr int kModeSample = 0;        // epilogue writes scores of sampled columns
constexpr int kModeFilter = 1;        // epilogue appends scores above the row threshold

// tcgen05.mma instruction descriptor: D fp32, A and B bf16, both K-major,
// M = 128, N = 256.
constexpr uint32_t kIdesc = f16_idesc(kBM, kBN);

// ---------------------------------------------------------------- arguments
// Work is split into units (KV head h, 128-row block rb, column segment seg):
// one CTA runs a unit's column tiles in order, so every output row has a
// fixed set of writers: 2 * nseg threads (segment x tile half). Writer slot
// = half * nseg + seg; slots 2j and 2j+1 share the j-th region of cap_pair
// entries of the row's list, one filling it upward from the start, the other
// downward from the end, so no writer needs an atomic. A pair whose two counts
// add up to more than cap_pair has overflowed (the row is re-selected).
struct GemmArgs {
    int r, hkv, nq, nq_pad, q_start;
    int nrb;               // row blocks per head = nq_pad / 128
    int ncol;              // column tiles of the longest row
    int nseg;              // column segments per row block (1, 2 or 4)
    int S;                 // key stride of the B operand's rows (sample stride, or 1)
    int stages;
    int a_slots;           // A tiles in flight (2 = the next unit's loads overlap this unit's MMAs)
    int nunits;            // hkv * nseg * nrb
    uint16_t* samp;        // sample mode: [rows, ld_samp] top 16 bits of the order keys (0 = none)
    long long ld_samp;
    const uint32_t* thr;   // filter mode: [rows] order-key thresholds
    unsigned* cnt;         // [rows, 2 * nseg] per-writer counts
    uint2* cand;           // [rows, ld_cand] (fp32 score bits, position)
    int cap_pair;          // entries per writer pair region
    long long ld_cand;     // entries per row = nseg * cap_pair
    unsigned* status;
    long long wait_limit;
};

struct Unit {
    int h, seg, rb;
    int c0, c1;            // active column tiles [c0, c1)
    long long pmin;        // position of the block's first query
};

// Units are ordered head, then segment, then row block: the CTAs running at
// one time work through the same key columns of one head and share them in L2.
__device__ __forceinline__ Unit decode_unit(int u, const GemmArgs& a) {
    Unit t;
    t.rb = u % a.nrb;
    const int rest = u / a.nrb;
    t.seg = rest % a.nseg;
    t.h = rest / a.nseg;
    const int qlast = min(t.rb * kBM + kBM - 1, a.nq - 1);
    const long long pmax = (long long)a.q_start + qlast;
    // the block's active tiles (those holding a column <= pmax), split evenly
    const int act = (int)min((long long)a.ncol, pmax / ((long long)kBN * a.S) + 1);
    t.c0 = (int)((long long)t.seg * act / a.nseg);
    t.c1 = (int)((long long)(t.seg + 1) * act / a.nseg);
    t.pmin = (long long)a.q_start + (long long)t.rb * kBM;
    return t;
}

// ---------------------------------------------------------------- score GEMM
// D[128 queries, 256 keys] = Qbar_h[rows] . Kt_h[cols]^T per tile, K = r.
// Shared memory: two A slots (one per unit, double-buffered), `stages` B
// stages, barriers.
template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rb = a.r * 2 < 128 ? (uint32_t)a.r * 2 : 128u;   // bytes per row in one swizzle atom
    const int atoms = a.r * 2 / (int)rb;
    const uint32_t a_bytes = (uint32_t)kBM * a.r * 2, b_bytes = (uint32_t)kBN * a.r * 2;
    uint8_t* Aslot = sm;
    uint8_t* Bst = sm + a.a_slots * a_bytes;
    float* stage_all = reinterpret_cast<float*>(Bst + a.stages * b_bytes);   // epilogue staging, kStageFloats per warp
    uint64_t* full = reinterpret_cast<uint64_t*>(stage_all + kEpiWarps * kStageFloats);
    uint64_t* empty = full + kMaxStages;
    uint64_t* afull = empty + kMaxStages;
    uint64_t* aempty = afull + 2;
    uint64_t* tfull = aempty + 2;
    uint64_t* tempty = tfull + 2;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&afull[i], 1);
            mbar_init(&aempty[i], 1);
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;

    auto fail = [&]() {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
    };
    // Every role loop is warp-uniform: lane 0 waits on the barrier and
    // broadcasts the outcome, lane 0 issues, the warp moves on together.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar, parity, a.wait_limit, abort_flag) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };

    // Issued asynchronous work, for the drain after an abort: TMA loads
    // (producer lane) and the last accumulator / A-slot commits (MMA lane).
    int a_issued = 0, b_issued = 0;
    int last_acc = -1, last_as = -1;
    uint32_t last_aph = 0, last_asph = 0;
    if (warp == 0) {   // ----------------------------------------------- TMA producer
        int it = 0, ui = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
            const Unit un = decode_unit(u, a);
            if (un.c1 <= un.c0) continue;
            const int as = ui % a.a_slots;
            if (!warp_wait(&aempty[as], ((uint32_t)(ui / a.a_slots) & 1u) ^ 1u)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&afull[as], a_bytes);
                for (int at = 0; at < atoms; ++at)
                    tma_load_2d(Aslot + as * a_bytes + at * kBM * rb, &tmA, at * 64, un.h * a.nq_pad + un.rb * kBM,
                                &afull[as]);
                a_issued = ui + 1;
            }
            __syncwarp();
            for (int c = un.c0; c < un.c1; ++c) {
                const int s = it % a.stages;
                const uint32_t ph = (uint32_t)(it / a.stages) & 1u;
                if (!warp_wait(&empty[s], ph ^ 1u)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t* Bs = Bst + s * b_bytes;
                    mbar_arrive_expect_tx(&full[s], b_bytes);
                    for (int at = 0; at < atoms; ++at)
                        tma_load_2d(Bs + at * kBN * rb, &tmB, un.h * a.r + at * 64, c * kBN, &full[s]);
                    b_issued = it + 1;
                }
                __syncwarp();
                ++it;
            }
            ++ui;
        }
        if (!ok && lane == 0) fail();
    } else if (warp == 1) {   // ---------------------------------------- MMA issuer
        const int nk = a.r / 16;
        int it = 0, ui = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
            const Unit un = decode_unit(u, a);
            if (un.c1 <= un.c0) continue;
            const int as = ui % a.a_slots;
            if (!warp_wait(&afull[as], (uint32_t)(ui / a.a_slots) & 1u)) {
                ok = false;
                break;
            }
            const uint32_t Asa = smem_addr(Aslot + as * a_bytes);
            for (int c = un.c0; c < un.c1; ++c) {
                const int s = it % a.stages;
                const uint32_t ph = (uint32_t)(it / a.stages) & 1u;
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!warp_wait(&tempty[acc], aph ^ 1u) || !warp_wait(&full[s], ph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t Bs = smem_addr(Bst + s * b_bytes);
                    const uint32_t d = tbase + (uint32_t)(acc * kBN);
                    for (int k = 0; k < nk; ++k) {
                        const uint32_t kb = (uint32_t)k * 32u;     // 16 bf16 of K per MMA
                        const uint32_t atom = kb / rb, within = kb % rb;
                        tc_mma(d, umma_desc(Asa + atom * kBM * rb + within, rb),
                               umma_desc(Bs + atom * kBN * rb + within, rb), kIdesc, k > 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                    tc_commit(&tfull[acc]);
                }
                __syncwarp();
                last_acc = acc;
                last_aph = aph;
                ++it;
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&aempty[as]);   // A slot free once this unit's MMAs are done
            __syncwarp();
            last_as = as;
            last_asph = (uint32_t)(ui / a.a_slots) & 1u;
            ++ui;
        }
        if (!ok && lane == 0) fail();
    } else if (warp >= kEpiWarp0) {   // ------------------------------- epilogue
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;   // TMEM lanes this warp may access
        const int half = ew >> 2;       // column half of the tile
        const int row_in = quarter * 32 + lane;
        float* stage = stage_all + ew * kStageFloats;
        int it = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
            const Unit un = decode_unit(u, a);
            const int q = un.rb * kBM + row_in;
            const bool vrow = q < a.nq;
            const int p = a.q_start + q;
            const long long grow = (long long)q * a.hkv + un.h;
            // filter mode: this thread's writer slot and list region
            const int slot = half * a.nseg + un.seg;
            const bool down = (slot & 1) != 0;
            // this writer's next list entry: upward from the region start, or
            // downward from its end (entries hold the raw fp32 score bits)
            uint2* wp = a.cand + grow * a.ld_cand + (long long)(slot >> 1) * a.cap_pair + (down ? a.cap_pair - 1 : 0);
            const int dir = down ? -1 : 1;
            float thr_f = 0.f;
            if (MODE == kModeFilter) thr_f = vrow ? key_floor(__ldg(&a.thr[grow])) : __int_as_float(0x7f800000);
            unsigned n = 0;
            for (int c = un.c0; c < un.c1; ++c) {
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!warp_wait(&tfull[acc], aph)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int col0 = c * kBN + half * 128;
                const uint32_t taddr = tbase + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * kBN + half * 128);
                for (int ch = 0; ch < 4; ch += 2) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(taddr + ch * 32, v0);
                    tmem_ld32(taddr + ch * 32 + 32, v1);
                    tmem_wait(v0);
                    tmem_wait(v1);
                    if (MODE == kModeSample) {
                        if (vrow) {
                            uint4* dst = reinterpret_cast<uint4*>(a.samp + grow * a.ld_samp + col0 + ch * 32);
#pragma unroll
                            for (int g = 0; g < 8; ++g) {
                                uint32_t w[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int j = g * 8 + e * 2;
                                    const uint32_t* src = j < 32 ? v0 : v1;
                                    const int jj = j & 31;
                                    const long long t0 = (long long)(col0 + ch * 32 + j) * a.S;
                                    const uint32_t k0 = t0 <= p ? score_key(__uint_as_float(src[jj])) >> 16 : 0u;
                                    const uint32_t k1 =
                                        t0 + a.S <= p ? score_key(__uint_as_float(src[jj + 1])) >> 16 : 0u;
                                    w[e] = k0 | (k1 << 16);
                                }
                                dst[g] = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    } else {
                        // Pass masks first (branch-free), then only the passing
                        // entries, read back from a per-warp staging tile.
                        const bool diag = (long long)(c + 1) * kBN - 1 > un.pmin;
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const uint32_t* v = k ? v1 : v0;
                            const int cb = col0 + ch * 32 + k * 32;   // first column of this chunk
                            uint32_t m = 0;
#pragma unroll
                            for (int j = 0; j < 32; ++j) m |= (__uint_as_float(v[j]) >= thr_f ? 1u : 0u) << j;
                            if (diag) {
                                const int lim = p - cb;   // columns cb + j with j <= lim are causal
                                m &= lim >= 31 ? 0xFFFFFFFFu : (lim < 0 ? 0u : (2u << lim) - 1u);
                            }
                            if (!vrow) m = 0;
                            if (__any_sync(0xffffffffu, m != 0u)) {
                                float4* st4 = reinterpret_cast<float4*>(stage + lane * kStageRow);
#pragma unroll
                                for (int g = 0; g < 8; ++g)
                                    st4[g] = make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                                         __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
                                __syncwarp();
                                // two passes per iteration: their shared-memory reads overlap
                                const uint32_t* srow = reinterpret_cast<const uint32_t*>(stage + lane * kStageRow);
                                while (m) {
                                    const int j1 = __ffs(m) - 1;
                                    m &= m - 1u;
                                    const int j2 = m ? __ffs(m) - 1 : j1;
                                    const bool two = m != 0u;
                                    if (two) m &= m - 1u;
                                    const uint32_t x1 = srow[j1], x2 = srow[j2];
                                    if (n < (unsigned)a.cap_pair) *wp = make_uint2(x1, (uint32_t)(cb + j1));
                                    wp += dir;
                                    ++n;
                                    if (two) {
                                        if (n < (unsigned)a.cap_pair) *wp = make_uint2(x2, (uint32_t)(cb + j2));
                                        wp += dir;
                                        ++n;
                                    }
                                }
                                __syncwarp();
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                ++it;
            }
            if (MODE == kModeFilter && ok && vrow) a.cnt[grow * kMaxSlots + slot] = n;
        }
        if (!ok && lane == 0) fail();
    }
    __syncthreads();
    if (*abort_flag) {
        // Every role has stopped and any abort is visible. Before shared
        // memory and TMEM are released, wait (with the fixed drain bound) for
        // the work already issued: each barrier has at most one outstanding
        // phase, its last issued one.
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < a.stages && s < b_issued; ++s) {
                const int last = s + ((b_issued - 1 - s) / a.stages) * a.stages;
                mbar_wait_bounded(&full[s], (uint32_t)(last / a.stages) & 1u, kDrainNs);
            }
            for (int s = 0; s < a.a_slots && s < a_issued; ++s) {
                const int last = s + ((a_issued - 1 - s) / a.a_slots) * a.a_slots;
                mbar_wait_bounded(&afull[s], (uint32_t)(last / a.a_slots) & 1u, kDrainNs);
            }
        }
        if (warp == 1 && lane == 0) {
            // MMAs complete in order: the last accumulator commit covers them all
            if (last_acc >= 0) mbar_wait_bounded(&tfull[last_acc], last_aph, kDrainNs);
            if (last_as >= 0) mbar_wait_bounded(&aempty[last_as], last_asph, kDrainNs);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kAccCols);
    }
}

// ---------------------------------------------------------------- group mean
// qb[h, q, c] = bf16(mean over the group of qt[q, h*G + g, c]); rows q >= nq zero.
__global__ void prefill_qbar_kernel(const uint16_t* __restrict__ qt, uint16_t* __restrict__ qb, int nq, int nq_pad,
                                    int hq, int hkv, int r) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)hkv * nq_pad * r;
    if (e >= total) return;
    const int c = (int)(e % r);
    const long long rest = e / r;
    const int q = (int)(rest % nq_pad);
    const int h = (int)(rest / nq_pad);
    const int G = hq / hkv;
    float s = 0.f;
    if (q < nq) {
        const uint16_t* src = qt + ((long long)q * hq + (long long)h * G) * r + c;
        for (int g = 0; g < G; ++g) s += __uint_as_float((uint32_t)src[(long long)g * r] << 16);
        s *= 1.0f / (float)G;
    }
    qb[e] = f2bf(s);
}

// ---------------------------------------------------------------- selection
struct SelArgs {
    int hkv, nq, nq_pad, q_start, B, cap, cap_pair, nseg, r, S, kth;
    long long rows, ld_samp, ld_cand;
    const uint16_t* samp;
    uint32_t* thr;
    const unsigned* cnt;
    const uint2* cand;
    const uint16_t* qb;
    const uint16_t* kt;
    int32_t* idx;
};

struct SelShared {
    BlockSelShared bs;
    int start[8], pre[9];
    int fb;
};

// In a 256-bin histogram, the bin b holding the rem-th largest entry, and the
// entries in bins above it (warp-wide; every lane gets the results).
__device__ __forceinline__ void warp_find_bin(const uint32_t* h, int rem, int lane, int* bin, int* above, int* total) {
    const int top = 255 - lane * 8;
    int s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += (int)h[top - j];
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    *total = __shfl_sync(0xffffffffu, incl, 31);
    const int excl = incl - s;
    int b = -1, ab = 0;
    if (excl < rem && rem <= incl) {
        int c = excl;
        for (int j = 0; j < 8; ++j) {
            const int hb = (int)h[top - j];
            if (c + hb >= rem) {
                b = top - j;
                ab = c;
                break;
            }
            c += hb;
        }
    }
    const unsigned m = __ballot_sync(0xffffffffu, b >= 0);
    const int src = m ? __ffs(m) - 1 : 0;
    *bin = __shfl_sync(0xffffffffu, b, src);
    *above = __shfl_sync(0xffffffffu, ab, src);
}

// theta_row (one warp per row) = the kth-largest 16-bit sampled key of the
// row, widened to 32 bits (so at least kth sampled keys are >= theta_row);
// rows short enough to keep every key, or with fewer than kth samples, get
// the smallest key, 1.
constexpr int kThrWarps = 8;
__global__ void __launch_bounds__(kThrWarps * 32) prefill_threshold_kernel(const SelArgs a) {
    __shared__ uint32_t hist[kThrWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kThrWarps + warp;
    if (row >= a.rows) return;
    const int q = (int)(row / a.hkv);
    const int p = a.q_start + q;
    if (p + 1 <= a.cap || a.samp == nullptr) {
        if (lane == 0) a.thr[row] = 1u;
        return;
    }
    const int ms = (int)min((long long)(p / a.S + 1), a.ld_samp);
    const uint16_t* src = a.samp + row * a.ld_samp;
    uint32_t* h = hist[warp];
    for (int i = lane; i < 256; i += 32) h[i] = 0u;
    __syncwarp();
    for (int i = lane; i < ms; i += 32) {
        const uint32_t k = src[i];
        if (k) atomicAdd(&h[k >> 8], 1u);
    }
    __syncwarp();
    int b1, ab1, total;
    warp_find_bin(h, a.kth, lane, &b1, &ab1, &total);
    if (total < a.kth) {
        if (lane == 0) a.thr[row] = 1u;
        return;
    }
    __syncwarp();
    for (int i = lane; i < 256; i += 32) h[i] = 0u;
    __syncwarp();
    for (int i = lane; i < ms; i += 32) {
        const uint32_t k = src[i];
        if ((k >> 8) == (uint32_t)b1) atomicAdd(&h[k & 255u], 1u);
    }
    __syncwarp();
    int b2, ab2, t2;
    warp_find_bin(h, a.kth - ab1, lane, &b2, &ab2, &t2);
    if (lane == 0) a.thr[row] = ((uint32_t)b1 << 24) | ((uint32_t)b2 << 16);
}

// Exact top-B of one row (dynamic shared memory: a bitmap of the row's
// positions, 4 * ceil((q_start + nq) / 32) bytes). The row's candidates are
// loaded once into registers (kSelItems per thread); longer lists are read
// from global memory on every pass, and rows re-done from scratch recompute
// their scores.
constexpr int kSelItems = 8;

__global__ void __launch_bounds__(kSelThreads) prefill_select_kernel(const SelArgs a) {
    __shared__ SelShared sh;
    __shared__ float sq[128];
    extern __shared__ uint32_t bitmap[];
    const int row = blockIdx.x;
    const int q = row / a.hkv, h = row % a.hkv;
    const int p = a.q_start + q;
    const int n = p + 1;
    const int need = min(a.B, n);
    const int slots = 2 * a.nseg;
    const uint2* cand = a.cand + (long long)row * a.ld_cand;
    int32_t* out = a.idx + (long long)row * a.B;
    if (threadIdx.x < 32) {   // writer counts -> list ranges, overflow check (warp 0)
        const int lane = threadIdx.x;
        const unsigned c = lane < slots ? __ldcg(&a.cnt[(long long)row * kMaxSlots + lane]) : 0u;
        const unsigned partner = __shfl_xor_sync(0xffffffffu, c, 1);
        const bool over = (lane < slots) && (lane & 1) && c + partner > (unsigned)a.cap_pair;
        const int cl = (int)min(c, (unsigned)a.cap_pair);
        int incl = cl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane < slots) {
            sh.start[lane] = (lane >> 1) * a.cap_pair + ((lane & 1) ? a.cap_pair - cl : 0);
            sh.pre[lane] = incl - cl;
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        const bool any_over = __any_sync(0xffffffffu, over);
        if (lane == 0) {
            sh.pre[slots] = tot;
            sh.fb = (any_over || tot < need) ? 1 : 0;
        }
    }
    __syncthreads();
    const bool fb = sh.fb != 0;
    const int items = sh.pre[slots];
    auto entry = [&](int i) -> uint2 {
        int j = 0;
        while (j + 1 < slots && i >= sh.pre[j + 1]) ++j;
        return __ldcg(&cand[sh.start[j] + (i - sh.pre[j])]);
    };
    if (!fb && items <= kSelThreads * kSelItems) {
        uint32_t kk[kSelItems], pp[kSelItems];
#pragma unroll
        for (int it = 0; it < kSelItems; ++it) {
            const int i = threadIdx.x + it * kSelThreads;
            kk[it] = 0u;
            pp[it] = 0u;
            if (i < items) {
                const uint2 e = entry(i);
                kk[it] = score_key(__uint_as_float(e.x));
                pp[it] = e.y;
            }
        }
        select_and_emit<kSelThreads>(
            [&](auto f) {
#pragma unroll
                for (int it = 0; it < kSelItems; ++it)
                    if (kk[it]) f(kk[it], pp[it]);
            },
            need, n, sh.bs, bitmap, out, a.B, [](int i) { return i; });
    } else if (!fb) {
        select_and_emit<kSelThreads>(
            [&](auto f) {
                for (int i = threadIdx.x; i < items; i += kSelThreads) {
                    const uint2 e = entry(i);
                    f(score_key(__uint_as_float(e.x)), e.y);
                }
            },
            need, n, sh.bs, bitmap, out, a.B, [](int i) { return i; });
    } else {
        // Re-done from scratch: scores recomputed on the CUDA cores (fp32 FMAs
        // over the r channels in order) for every causal position.
        const int r = a.r;
        for (int c = threadIdx.x; c < r; c += kSelThreads)
            sq[c] = __uint_as_float((uint32_t)a.qb[((long long)h * a.nq_pad + q) * r + c] << 16);
        __syncthreads();
        auto recompute = [&](int t) -> uint32_t {
            const uint4* kr = reinterpret_cast<const uint4*>(a.kt + ((long long)t * a.hkv + h) * r);
            float acc = 0.f;
            for (int c8 = 0; c8 < r / 8; ++c8) {
                const uint4 w = __ldg(kr + c8);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc = fmaf(sq[c8 * 8 + 2 * j], bf16lo(ws[j]), acc);
                    acc = fmaf(sq[c8 * 8 + 2 * j + 1], bf16hi(ws[j]), acc);
                }
            }
            return score_key(acc);
        };
        select_and_emit<kSelThreads>(
            [&](auto f) {
                for (int t = threadIdx.x; t < n; t += kSelThreads) f(recompute(t), (uint32_t)t);
            },
            need, n, sh.bs, bitmap, out, a.B, [](int i) { return i; });
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

// 2-D bf16 tensor map: `outer` rows of `inner` elements, rows `row_bytes`
// apart; boxes of box_inner x box_outer, swizzled to the box's row width.
bool make_tensor_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const uint32_t bytes = box_inner * 2;
    const CUtensorMapSwizzle sw = bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

PrefillPlan plan_prefill(int hq, int hkv, int r, int T, int nq, int B) {
    PrefillPlan P{};
    (void)hq;
    P.nq_pad = (nq + kBM - 1) / kBM * kBM;
    P.rows = (long long)nq * hkv;
    // Sample stride: about 64 samples per B keys, at most kMaxSamples per row.
    int S = 1;
    while (S * 2 <= B / 64) S *= 2;
    while (((long long)T + S - 1) / S > kMaxSamples) S *= 2;
    P.S = S;
    P.kth = (int)((5LL * B + 4LL * S - 1) / (4LL * S)) + 16;    // ceil(1.25 B / S) + 16
    const long long expect = (long long)P.kth * S;               // keys expected above theta
    long long cap = 2 * expect;
    if (cap < B + B / 2 + 512) cap = B + B / 2 + 512;
    if (cap < 2048) cap = 2048;
    P.cap = (int)((cap + 255) / 256 * 256);
    P.sample = T > P.cap;
    const long long m = ((long long)T + S - 1) / S;
    P.ncol_sample = (int)((m + kBN - 1) / kBN);
    P.ld_samp = (long long)P.ncol_sample * kBN;
    const size_t a_bytes = (size_t)kBM * r * 2, b_bytes = (size_t)kBN * r * 2;
    const size_t staging = (size_t)kEpiWarps * kStageFloats * 4;
    const size_t fixed = (2 * kMaxStages + 8) * 8 + 16 + 1024;   // barriers, TMEM slot, alignment slack
    const size_t budget = 227 * 1024 - fixed - staging;
    int a_slots = 2;
    long long stages = ((long long)budget - 2 * (long long)a_bytes) / (long long)b_bytes;
    if (stages < 3) {
        a_slots = 1;
        stages = ((long long)budget - (long long)a_bytes) / (long long)b_bytes;
    }
    if (stages > kMaxStages) stages = kMaxStages;
    P.stages = (int)stages;
    P.a_slots = a_slots;
    size_t smem = a_slots * a_bytes + P.stages * b_bytes + staging + fixed;
    if (smem < 120 * 1024) smem = 120 * 1024;   // one CTA per SM: each holds all 512 TMEM columns
    P.gemm_smem = (int)smem;
    size_t off = 0;
    P.off_qb = off;
    off = align256(off + (size_t)hkv * P.nq_pad * r * 2);
    P.off_samp = off;
    if (P.sample) off = align256(off + (size_t)P.rows * P.ld_samp * 2);
    P.off_thr = off;
    off = align256(off + (size_t)P.rows * 4);
    P.off_cnt = off;
    off = align256(off + (size_t)P.rows * kMaxSlots * 4);
    P.off_cand = off;
    off = align256(off + (size_t)P.rows * 2 * P.cap * 8);   // room for the 4-segment layout
    P.bytes = off;
    return P;
}

cudaError_t launch_prefill_index(const LaunchCtx& ctx, const PrefillPlan& P, const uint16_t* qt, const uint16_t* kt,
                                 int hq, int hkv, int r, int T, int nq, int q_start, int B, int32_t* idx, uint8_t* ws,
                                 unsigned* status) {
    uint16_t* qb = reinterpret_cast<uint16_t*>(ws + P.off_qb);
    uint16_t* samp = P.sample ? reinterpret_cast<uint16_t*>(ws + P.off_samp) : nullptr;
    uint32_t* thr = reinterpret_cast<uint32_t*>(ws + P.off_thr);
    unsigned* cnt = reinterpret_cast<unsigned*>(ws + P.off_cnt);
    uint2* cand = reinterpret_cast<uint2*>(ws + P.off_cand);
    const long long pmax = (long long)q_start + nq - 1;

    {
        const long long total = (long long)hkv * P.nq_pad * r;
        prefill_qbar_kernel<<<(unsigned)((total + 255) / 256), 256, 0, ctx.stream>>>(qt, qb, nq, P.nq_pad, hq, hkv, r);
    }
    CUtensorMap mA, mB, mS;
    const uint32_t box_in = r < 64 ? (uint32_t)r : 64u;
    if (!make_tensor_map_2d(&mA, qb, (uint64_t)r, (uint64_t)hkv * P.nq_pad, (uint64_t)r * 2, box_in, kBM) ||
        !make_tensor_map_2d(&mB, kt, (uint64_t)hkv * r, (uint64_t)T, (uint64_t)hkv * r * 2, box_in, kBN))
        return cudaErrorInvalidValue;
    const long long nsamp_rows = ((long long)T + P.S - 1) / P.S;
    const bool any_sample = P.sample && pmax + 1 > P.cap;
    if (any_sample &&
        !make_tensor_map_2d(&mS, kt, (uint64_t)hkv * r, (uint64_t)nsamp_rows, (uint64_t)hkv * r * 2 * P.S, box_in, kBN))
        return cudaErrorInvalidValue;

    GemmArgs g{};
    g.r = r;
    g.hkv = hkv;
    g.nq = nq;
    g.nq_pad = P.nq_pad;
    g.q_start = q_start;
    g.nrb = P.nq_pad / kBM;
    g.stages = P.stages;
    g.a_slots = P.a_slots;
    g.thr = thr;
    g.cnt = cnt;
    g.cand = cand;
    g.status = status;
    g.wait_limit = ctx.wait_limit;

    // Filter pass layout: 4 column segments per row block when rows span many
    // tiles (enough units to fill the GPU), else 2 or 1.
    const int ncol_f = (int)((pmax + 1 + kBN - 1) / kBN);
    const int nseg = ncol_f >= 16 ? 4 : (ncol_f >= 2 ? 2 : 1);
    const int cap_pair = nseg == 1 ? P.cap : P.cap / 2;

    SelArgs s{};
    s.hkv = hkv;
    s.nq = nq;
    s.nq_pad = P.nq_pad;
    s.q_start = q_start;
    s.B = B;
    s.cap = P.cap;
    s.cap_pair = cap_pair;
    s.nseg = nseg;
    s.r = r;
    s.S = P.S;
    s.kth = P.kth;
    s.rows = P.rows;
    s.ld_samp = P.ld_samp;
    s.ld_cand = (long long)nseg * cap_pair;
    s.samp = any_sample ? samp : nullptr;
    s.thr = thr;
    s.cnt = cnt;
    s.cand = cand;
    s.qb = qb;
    s.kt = kt;
    s.idx = idx;

    cudaError_t e;
    if (any_sample) {
        GemmArgs gs = g;
        gs.S = P.S;
        gs.ncol = (int)((pmax / P.S + 1 + kBN - 1) / kBN);
        gs.nseg = 1;
        gs.nunits = hkv * gs.nrb;
        gs.samp = samp;
        gs.ld_samp = P.ld_samp;
        if ((e = ensure_dyn_smem((const void*)prefill_gemm_kernel<kModeSample>, P.gemm_smem)) != cudaSuccess) return e;
        const unsigned grid = (unsigned)(gs.nunits < ctx.num_sms ? gs.nunits : ctx.num_sms);
        prefill_gemm_kernel<kModeSample><<<grid, kGemmThreads, P.gemm_smem, ctx.stream>>>(mA, mS, gs);
    }
    prefill_threshold_kernel<<<(unsigned)((P.rows + kThrWarps - 1) / kThrWarps), kThrWarps * 32, 0, ctx.stream>>>(s);
    {
        GemmArgs gf = g;
        gf.S = 1;
        gf.ncol = ncol_f;
        gf.nseg = nseg;
        gf.nunits = hkv * nseg * gf.nrb;
        gf.cap_pair = cap_pair;
        gf.ld_cand = (long long)nseg * cap_pair;
        if ((e = ensure_dyn_smem((const void*)prefill_gemm_kernel<kModeFilter>, P.gemm_smem)) != cudaSuccess) return e;
        const unsigned grid = (unsigned)(gf.nunits < ctx.num_sms ? gf.nunits : ctx.num_sms);
        prefill_gemm_kernel<kModeFilter><<<grid, kGemmThreads, P.gemm_smem, ctx.stream>>>(mA, mB, gf);
    }
    {
        const int nw = (int)((pmax + 1 + 31) / 32);
        const int smem = nw * 4;
        if ((e = ensure_dyn_smem((const void*)prefill_select_kernel, smem)) != cudaSuccess) return e;
        prefill_select_kernel<<<(unsigned)P.rows, kSelThreads, smem, ctx.stream>>>(s);
    }
    return cudaGetLastError();
}

}  // namespace lsa
