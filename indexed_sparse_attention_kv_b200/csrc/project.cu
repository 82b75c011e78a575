// Scoring preparation: projection onto the per-KV-head scoring subspace, and
// incremental block centroids.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Fig. 1
// (queries and keys scored in a shared low-dimensional subspace) and Fig. 9
// ("scoring preparation": the key projection that fills the projected-key
// cache, reported as a negligible share of the step). Every KV head h has a
// basis P[h] of r vectors of length d; a key of head h and the query heads of
// h's group project onto it: y[b, t, i, j] = <P[i / G, j], x[b, t, i]>.
// LongCat Sparse Attention, Abstract, strategy (3) Hierarchical Indexing: the
// coarse stage scores block centroids, which an append keeps current.
//
// The projection is a dense contraction (per row 2 d r flops against 2 d
// bytes in, r bytes or 2 r bytes out: about 43 flop/byte at d = 128, r = 64),
// above what the CUDA cores sustain at HBM speed, so it runs on the tensor
// cores: a persistent tcgen05 GEMM, D[128 rows, r] = X_i[rows, d] . P[i/G]^T,
// with X tiles and the basis staged by TMA in swizzled shared memory and two
// fp32 accumulators in TMEM. Warp 0 issues the TMA loads, warp 1 the MMAs,
// warps 2..5 drain TMEM (one 32-lane quarter each), round to bf16 or FP8
// E4M3 and store whole output rows.
#include <cuda.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {
namespace {

constexpr int kPM = 128;                 // rows per tile = TMEM lanes
constexpr int kProjThreads = 192;        // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2..5 epilogue
constexpr int kProjEpiWarp0 = 2;
constexpr int kProjEpiWarps = 4;
constexpr int kProjMaxStages = 6;

struct ProjArgs {
    uint8_t* y;               // [rows, H, r] bf16 or e4m3
    int H, G, d, r, nk;       // nk = d / 16 k-steps
    int rb, atoms;            // bytes per swizzled row of a tile atom, atoms across d
    int nseq;                 // independent row ranges (sequences)
    long long seq_rows;       // rows between consecutive sequences' ranges (T)
    long long row0;           // first row of sequence 0's range (t0)
    int len;                  // rows per range (n)
    int tiles_per_seq;        // ceil(len / 128)
    long long ntiles;         // H * nseq * tiles_per_seq
    int stages;
    uint32_t acc_cols;        // TMEM columns allocated (two accumulators of r)
    unsigned* status;
    long long wait_limit;
};

struct Tile {
    int head, basis;
    long long z0;             // first row of the tile
    int valid;                // rows of the tile inside its range
};

// Tiles are ordered head-major, so a CTA's contiguous share of them changes
// basis rarely.
__device__ __forceinline__ Tile decode_tile(long long u, const ProjArgs& a) {
    Tile t;
    const long long per_head = (long long)a.nseq * a.tiles_per_seq;
    t.head = (int)(u / per_head);
    const long long rem = u - (long long)t.head * per_head;
    const int s = (int)(rem / a.tiles_per_seq);
    const int k = (int)(rem - (long long)s * a.tiles_per_seq);
    t.basis = t.head / a.G;
    t.z0 = (long long)s * a.seq_rows + a.row0 + (long long)k * kPM;
    const int left = a.len - k * kPM;
    t.valid = left < kPM ? left : kPM;
    return t;
}

template <bool FP8>
__global__ void __launch_bounds__(kProjThreads, 1)
    project_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                   const ProjArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t x_bytes = (uint32_t)(kPM * a.rb * a.atoms);
    const uint32_t p_bytes = (uint32_t)(a.r * a.rb * a.atoms);
    uint8_t* Xst = sm;
    uint8_t* Pslot = Xst + a.stages * x_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(Pslot + 2 * p_bytes);
    uint64_t* empty = full + kProjMaxStages;
    uint64_t* pfull = empty + kProjMaxStages;
    uint64_t* pempty = pfull + 2;
    uint64_t* tfull = pempty + 2;
    uint64_t* tempty = tfull + 2;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

    const long long u0 = (long long)blockIdx.x * a.ntiles / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * a.ntiles / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], 1);
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kProjEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, a.acc_cols);
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
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(bar, parity, a.wait_limit, abort_flag) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };

    // Issued asynchronous work, for the drain after an abort: TMA loads
    // (producer lane) and the last accumulator / basis-slot commits (MMA lane).
    long long x_issued = 0;
    int p_issued = 0, last_acc = -1, last_ps = -1;
    uint32_t last_aph = 0, last_psph = 0;
    if (warp == 0) {   // ----------------------------------------------- TMA producer
        int pi = -1, cur_basis = -1;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const Tile t = decode_tile(u, a);
            if (t.basis != cur_basis) {   // the basis of the next run of tiles into the other slot
                ++pi;
                cur_basis = t.basis;
                const int ps = pi & 1;
                if (!warp_wait(&pempty[ps], ((uint32_t)(pi >> 1) & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&pfull[ps], p_bytes);
                    for (int at = 0; at < a.atoms; ++at)
                        tma_load_2d(Pslot + ps * p_bytes + at * a.r * a.rb, &tmP, at * (a.rb / 2), t.basis * a.r,
                                    &pfull[ps]);
                    p_issued = pi + 1;
                }
                __syncwarp();
            }
            const long long it = u - u0;
            const int s = (int)(it % a.stages);
            const uint32_t ph = (uint32_t)(it / a.stages) & 1u;
            if (!warp_wait(&empty[s], ph ^ 1u)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], x_bytes);
                for (int at = 0; at < a.atoms; ++at)
                    tma_load_2d(Xst + s * x_bytes + at * kPM * a.rb, &tmX, t.head * a.d + at * (a.rb / 2),
                                (int)t.z0, &full[s]);
                x_issued = it + 1;
            }
            __syncwarp();
        }
        if (!ok && lane == 0) fail();
    } else if (warp == 1) {   // ---------------------------------------- MMA issuer
        const uint32_t idesc = f16_idesc(kPM, a.r);
        int pi = -1, cur_basis = -1;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const Tile t = decode_tile(u, a);
            if (t.basis != cur_basis) {
                if (pi >= 0 && lane == 0) tc_commit(&pempty[pi & 1]);   // previous basis free after its MMAs
                __syncwarp();
                if (pi >= 0) {
                    last_ps = pi & 1;
                    last_psph = (uint32_t)(pi >> 1) & 1u;
                }
                ++pi;
                cur_basis = t.basis;
                if (!warp_wait(&pfull[pi & 1], (uint32_t)(pi >> 1) & 1u)) {
                    ok = false;
                    break;
                }
            }
            const long long it = u - u0;
            const int s = (int)(it % a.stages);
            const uint32_t ph = (uint32_t)(it / a.stages) & 1u;
            const int acc = (int)(it & 1);
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            if (!warp_wait(&tempty[acc], aph ^ 1u) || !warp_wait(&full[s], ph)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t Xs = smem_addr(Xst + s * x_bytes);
                const uint32_t Ps = smem_addr(Pslot + (pi & 1) * p_bytes);
                const uint32_t dcol = tbase + (uint32_t)(acc * a.r);
                for (int k = 0; k < a.nk; ++k) {
                    const uint32_t kb = (uint32_t)k * 32u;   // 16 bf16 of K per MMA
                    const uint32_t atom = kb / (uint32_t)a.rb, within = kb % (uint32_t)a.rb;
                    tc_mma(dcol, umma_desc(Xs + atom * kPM * a.rb + within, a.rb),
                           umma_desc(Ps + atom * a.r * a.rb + within, a.rb), idesc, k > 0 ? 1u : 0u);
                }
                tc_commit(&empty[s]);
                tc_commit(&tfull[acc]);
            }
            __syncwarp();
            last_acc = acc;
            last_aph = aph;
        }
        if (!ok && lane == 0) fail();
    } else if (warp >= kProjEpiWarp0) {   // ------------------------- epilogue
        const int quarter = warp & 3;     // TMEM lanes this warp may access
        const int row_in = quarter * 32 + lane;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const Tile t = decode_tile(u, a);
            const long long it = u - u0;
            const int acc = (int)(it & 1);
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            if (!warp_wait(&tfull[acc], aph)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool vrow = row_in < t.valid;
            const long long orow = ((t.z0 + row_in) * a.H + t.head) * a.r;   // output element offset
            const uint32_t taddr = tbase + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * a.r);
            for (int c0 = 0; c0 < a.r; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + c0, v);
                tmem_wait16(v);
                if (vrow) {
                    if (FP8) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                                make_float2(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1])), __NV_SATFINITE,
                                __NV_E4M3);
                            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                                make_float2(__uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])),
                                __NV_SATFINITE, __NV_E4M3);
                            w[j] = (uint32_t)lo | ((uint32_t)hi << 16);
                        }
                        *reinterpret_cast<uint4*>(a.y + orow + c0) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else {
                        uint32_t w[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            w[j] = (uint32_t)f2bf(__uint_as_float(v[2 * j])) |
                                   ((uint32_t)f2bf(__uint_as_float(v[2 * j + 1])) << 16);
                        uint4* dst = reinterpret_cast<uint4*>(a.y + (orow + c0) * 2);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
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
            for (int s = 0; s < a.stages && s < x_issued; ++s) {
                const long long last = s + ((x_issued - 1 - s) / a.stages) * a.stages;
                mbar_wait_bounded(&full[s], (uint32_t)(last / a.stages) & 1u, kDrainNs);
            }
            for (int s = 0; s < 2 && s < p_issued; ++s) {
                const int last = s + ((p_issued - 1 - s) / 2) * 2;
                mbar_wait_bounded(&pfull[s], (uint32_t)(last >> 1) & 1u, kDrainNs);
            }
        }
        if (warp == 1 && lane == 0) {
            // MMAs complete in order: the last accumulator commit covers them all
            if (last_acc >= 0) mbar_wait_bounded(&tfull[last_acc], last_aph, kDrainNs);
            if (last_ps >= 0) mbar_wait_bounded(&pempty[last_ps], last_psph, kDrainNs);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, a.acc_cols);
    }
}

// ---------------------------------------------------------------- centroids
// One thread per (sequence, touched block, head, component): the block's
// new tokens in position order, c <- bf16(c + kt[t]) after every add. The
// fp32 sum of two bf16 values rounds to the same bf16 as their exact sum.
__global__ void centroid_update_kernel(const uint16_t* __restrict__ kt, uint16_t* __restrict__ cen, int T, int hkv,
                                       int r, int blk, int t0, int n, int j0, int nj, int nblk, long long total) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const long long per_b = (long long)nj * hkv * r;
    const int b = (int)(e / per_b);
    long long rem = e - (long long)b * per_b;
    const int jj = (int)(rem / ((long long)hkv * r));
    rem -= (long long)jj * hkv * r;
    const int h = (int)(rem / r), c = (int)(rem - (long long)h * r);
    const int j = j0 + jj;
    const int ta = max(t0, j * blk), tb = min(t0 + n, (j + 1) * blk);
    const size_t ci = (((size_t)b * nblk + j) * hkv + h) * r + c;
    float s = bf16lo(cen[ci]);
    for (int t = ta; t < tb; ++t)
        s = bf16lo(f2bf(s + bf16lo(kt[(((size_t)b * T + t) * hkv + h) * r + c])));
    cen[ci] = f2bf(s);
}

size_t project_fixed_smem(size_t p_bytes) { return 2 * p_bytes + (2 * kProjMaxStages + 8) * 8 + 16 + 1024; }

}  // namespace

// X stages that fit next to two basis slots in 220 KB of shared memory (at
// most kProjMaxStages, no more than the tiles); below 2 the shape is not supported.
int project_stages(int d, int r, long long ntiles) {
    const int rb = d * 2 >= 128 ? 128 : d * 2;
    const int atoms = (d * 2 + rb - 1) / rb;
    const size_t x_bytes = (size_t)kPM * rb * atoms, p_bytes = (size_t)r * rb * atoms;
    const size_t fixed = project_fixed_smem(p_bytes);
    if (fixed >= 220u * 1024u) return 0;
    long long st = (long long)((220u * 1024u - fixed) / x_bytes);
    if (st > kProjMaxStages) st = kProjMaxStages;
    if (st >= 2 && st > ntiles) st = ntiles < 2 ? 2 : ntiles;
    return (int)st;
}

cudaError_t launch_project(const LaunchCtx& ctx, const uint16_t* x, const uint16_t* P, void* y, bool fp8, int batch,
                           int T, int H, int d, int r, int nbases, int t0, int n, unsigned* status) {
    if (n == 0) return cudaSuccess;
    ProjArgs a{};
    a.y = static_cast<uint8_t*>(y);
    a.H = H;
    a.G = H / nbases;
    a.d = d;
    a.r = r;
    a.nk = d / 16;
    a.rb = d * 2 >= 128 ? 128 : d * 2;
    a.atoms = (d * 2 + a.rb - 1) / a.rb;
    // a range covering whole sequences is one range over all rows
    if (t0 == 0 && n == T) {
        a.nseq = 1;
        a.seq_rows = 0;
        a.row0 = 0;
        a.len = batch * T;
    } else {
        a.nseq = batch;
        a.seq_rows = T;
        a.row0 = t0;
        a.len = n;
    }
    a.tiles_per_seq = (a.len + kPM - 1) / kPM;
    a.ntiles = (long long)H * a.nseq * a.tiles_per_seq;
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * r)) cols <<= 1;
    a.acc_cols = cols;
    a.status = status;
    a.wait_limit = ctx.wait_limit;
    const size_t x_bytes = (size_t)kPM * a.rb * a.atoms, p_bytes = (size_t)r * a.rb * a.atoms;
    const size_t fixed = project_fixed_smem(p_bytes);
    const int stages = project_stages(d, r, a.ntiles);
    if (stages < 2) return cudaErrorInvalidValue;
    a.stages = stages;
    // at least 120 KB, so that one CTA runs per SM and TMEM allocations never
    // wait on a neighbour
    size_t smem = (size_t)stages * x_bytes + fixed;
    if (smem < 120u * 1024u) smem = 120u * 1024u;

    CUtensorMap mX, mP;
    const uint32_t box_in = (uint32_t)(a.rb / 2);
    if (!make_tensor_map_2d(&mX, x, (uint64_t)H * d, (uint64_t)batch * T, (uint64_t)H * d * 2, box_in, kPM) ||
        !make_tensor_map_2d(&mP, P, (uint64_t)d, (uint64_t)nbases * r, (uint64_t)d * 2, box_in, (uint32_t)r))
        return cudaErrorInvalidValue;
    auto kern = fp8 ? project_kernel<true> : project_kernel<false>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    long long grid = a.ntiles < ctx.num_sms ? a.ntiles : ctx.num_sms;
    kern<<<(unsigned)grid, kProjThreads, smem, ctx.stream>>>(mX, mP, a);
    return cudaGetLastError();
}

cudaError_t launch_centroid_update(const LaunchCtx& ctx, const uint16_t* kt, uint16_t* cen, int batch, int T, int hkv,
                                   int r, int blk, int t0, int n) {
    if (n == 0) return cudaSuccess;
    const int nblk = (T + blk - 1) / blk;
    const int j0 = t0 / blk, j1 = (t0 + n - 1) / blk;
    const int nj = j1 - j0 + 1;
    const long long total = (long long)batch * nj * hkv * r;
    const int threads = 256;
    const long long blocks = (total + threads - 1) / threads;
    centroid_update_kernel<<<(unsigned)blocks, threads, 0, ctx.stream>>>(kt, cen, T, hkv, r, blk, t0, n, j0, nj,
                                                                        nblk, total);
    return cudaGetLastError();
}

}  // namespace lsa
