// Deterministic top-B selection per row with a thread-block-cluster radix select.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Fig. 1:
// each KV head keeps the B token positions with the largest scores. Ties at
// the threshold go to the lower position; the set is written in ascending order
// and padded with -1 when fewer than B candidates (non-NaN scores) exist.
//
// Scores map to order-preserving 32-bit keys (NaN -> 0, never selected). One
// cluster of CS CTAs owns a row, CTA k a contiguous segment of it, warp w of a
// CTA a contiguous sub-range of that segment.
//   1. The histogram of the top 11 key bits of the whole row: either built by
//      the scorer while it wrote the scores (decode path), or here, per CTA in
//      shared memory and summed over the cluster through distributed shared
//      memory. From it, the bin b0 holding the B-th largest key.
//   2. One pass over the keys in position order: every warp appends the
//      (key, position) pairs of bin >= b0 to its own list (about B plus the
//      threshold bin's keys per row: a small fraction of the row).
//   3. The keys of bin b0 of the whole cluster are gathered in every CTA and two
//      local radix passes give the exact threshold key theta and the number of
//      ties at theta to take.
//   4. Counts above / at theta per warp, exclusive prefix sums over warps and
//      over the cluster's CTAs, and a ballot compaction of the short lists write
//      the positions in ascending order.
// Whenever a list or the threshold bin is too large for shared memory (e.g.
// many equal scores), the cluster switches, uniformly, to radix passes and a
// compaction over the keys themselves, with the same result.
#include <cooperative_groups.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace cg = cooperative_groups;

namespace lsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins = 2048;
constexpr int kListPerWarp = 256;                       // (key, position) entries per warp
constexpr int kListCap = kListPerWarp * kTopkWarps;     // per CTA
constexpr int kGatherCap = 4096;                        // bin-b0 keys of the whole cluster
constexpr int kMaxCluster = 8;
constexpr int kBatch = 8;                               // 128-key steps whose loads are issued together

struct TopkArgs {
    const float* scores;      // [rows, n]
    int32_t* idx;             // [rows, B]
    const int32_t* blkmap;    // optional [rows, keep]: candidate c -> blkmap[c / blk] * blk + c % blk
    uint32_t* ghist;          // optional [rows, kBins] histogram of key >> 21; zeroed here after use
    int n, B, seg, blk, keep;
};

struct TopkShared {
    uint32_t red[kBins];            // row histogram
    uint32_t hist[kBins];           // this CTA's histogram / local refinement histogram
    uint32_t lkey[kListCap];        // per-warp lists (position order) of keys in bins >= b0
    int lpos[kListCap];
    uint32_t cand[kListCap];        // this CTA's bin-b0 keys (any order)
    uint32_t gathered[kGatherCap];  // the cluster's bin-b0 keys
    int wlist[kTopkWarps], wb0[kTopkWarps];
    int scan[kTopkWarps];
    int warp_gt[kTopkWarps], warp_eq[kTopkWarps];
    int warp_sel_before[kTopkWarps], warp_eq_before[kTopkWarps];
    int cta_gt, cta_eq, ncand, overflow;
    uint32_t bstar;
    int above;
    int total;
};

// Exclusive prefix sum over the CTA's threads (thread order); returns the
// exclusive prefix, and the CTA total through *total.
__device__ __forceinline__ int block_excl_scan(int v, int* scan, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scan[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kTopkWarps ? scan[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kTopkWarps) scan[lane] = w;   // inclusive per warp
    }
    __syncthreads();
    const int warp_excl = warp ? scan[warp - 1] : 0;
    const int res = warp_excl + x - v;
    *total = scan[kTopkWarps - 1];
    __syncthreads();
    return res;
}

// Warp-level exclusive prefix sum; *total = the warp's sum.
__device__ __forceinline__ int warp_excl_scan(int v, int* total) {
    const int lane = threadIdx.x & 31;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    *total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
}

// Given histogram `red` (nb bins) find the bin holding the krem-th largest
// element counted from the top; sets sh.bstar and sh.above (count above it)
// and returns the histogram total. All threads must call it.
__device__ __forceinline__ int find_bin(const uint32_t* red, int nb, int krem, TopkShared& sh) {
    const int per = nb / kTopkThreads;
    const int hi = nb - 1 - (int)threadIdx.x * per;
    int local = 0;
    for (int q = 0; q < per; ++q) local += (int)red[hi - q];
    int total;
    const int above_me = block_excl_scan(local, sh.scan, &total);
    if (above_me < krem && krem <= above_me + local) {
        int cum = above_me;
        for (int q = 0; q < per; ++q) {
            const int c = (int)red[hi - q];
            if (cum + c >= krem) {
                sh.bstar = (uint32_t)(hi - q);
                sh.above = cum;
                break;
            }
            cum += c;
        }
    }
    __syncthreads();
    return total;
}

// Sum histogram `h` (nb <= kBins bins) over the cluster's CTAs into `red`; all
// of a thread's remote loads are independent and in flight together.
__device__ __forceinline__ void cluster_reduce(cg::cluster_group& cluster, uint32_t* h, uint32_t* red, int nb, int CS) {
    constexpr int kPer = kBins / kTopkThreads;
    uint32_t v[kPer][kMaxCluster];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int bin = q * kTopkThreads + threadIdx.x;
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr)
            v[q][rr] = (rr < CS && bin < nb) ? cluster.map_shared_rank(h, rr)[bin] : 0u;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int bin = q * kTopkThreads + threadIdx.x;
        uint32_t s = 0;
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) s += v[q][rr];
        if (bin < nb) red[bin] = s;
    }
}

// The 4 keys at sub-range positions i .. i+3 (i a multiple of 4) of a warp
// range ending at `end`; 16-byte loads when the row is 16-byte aligned.
__device__ __forceinline__ void load4(const float* src, bool vec, int i, int end, uint32_t k[4]) {
    if (vec && i + 3 < end) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src + i));
        k[0] = score_key(v.x);
        k[1] = score_key(v.y);
        k[2] = score_key(v.z);
        k[3] = score_key(v.w);
    } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) k[u] = i + u < end ? score_key(__ldcg(src + i + u)) : 0u;
    }
}

template <bool EXT_HIST>
__global__ void __launch_bounds__(kTopkThreads) topk_cluster_kernel(const TopkArgs a) {
    cg::cluster_group cluster = cg::this_cluster();
    const int CS = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    extern __shared__ __align__(16) uint8_t topk_smem[];
    TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);

    const int base = rank * a.seg;
    int len = a.n - base;
    len = len < 0 ? 0 : (len > a.seg ? a.seg : len);
    const float* src = a.scores + (size_t)row * a.n + base;
    const bool vec = (a.n & 3) == 0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_launch_dependents();
    pdl_wait();   // the scores (and histogram) come from the previous kernel
    // warp sub-range of the segment, a multiple of 128 keys (4 per lane per step)
    int wlen = (len + kTopkWarps - 1) / kTopkWarps;
    wlen = (wlen + 127) & ~127;
    const int wbeg = min(len, warp * wlen), wend = min(len, wbeg + wlen);

    // ---- 1. row histogram of key >> 21 and the threshold bin b0
    if (EXT_HIST) {
        for (int i = tid; i < kBins; i += kTopkThreads) sh.red[i] = a.ghist[(size_t)row * kBins + i];
        __syncthreads();
    } else {
        for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int i00 = wbeg; i00 < wend; i00 += 128 * kBatch) {
            uint32_t kk[kBatch][4];
#pragma unroll
            for (int ub = 0; ub < kBatch; ++ub) load4(src, vec, i00 + ub * 128 + lane * 4, wend, kk[ub]);
#pragma unroll
            for (int ub = 0; ub < kBatch; ++ub)
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (kk[ub][u]) atomicAdd(&sh.hist[kk[ub][u] >> 21], 1u);
        }
        cluster.sync();
        cluster_reduce(cluster, sh.hist, sh.red, kBins, CS);
        __syncthreads();
    }
    int krem = a.B;
    const int total = find_bin(sh.red, kBins, krem, sh);
    const bool take_all = total <= a.B;
    const uint32_t b0 = take_all ? 0u : sh.bstar;
    if (!take_all) krem -= sh.above;
    const int in_b0 = take_all ? 0 : (int)sh.red[b0];

    // ---- 2. per-warp lists of (key, position) with bin >= b0, in position order
    uint32_t* wkey = sh.lkey + warp * kListPerWarp;
    int* wpos = sh.lpos + warp * kListPerWarp;
    int wc = 0;
    for (int i00 = wbeg; i00 < wend; i00 += 128 * kBatch) {
        uint32_t kk[kBatch][4];   // all loads of the batch in flight before any use
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) load4(src, vec, i00 + ub * 128 + lane * 4, wend, kk[ub]);
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) {
            const int i = i00 + ub * 128 + lane * 4;
            bool f[4];
            int c = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                f[u] = kk[ub][u] != 0u && (kk[ub][u] >> 21) >= b0;
                c += f[u];
            }
            int tot;
            int slot = wc + warp_excl_scan(c, &tot);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (f[u]) {
                    if (slot < kListPerWarp) {
                        wkey[slot] = kk[ub][u];
                        wpos[slot] = base + i + u;
                    }
                    ++slot;
                }
            }
            wc += tot;
        }
    }
    if (lane == 0) sh.wlist[warp] = wc;
    __syncthreads();
    bool over = false;
    for (int w = 0; w < kTopkWarps; ++w) over |= sh.wlist[w] > kListPerWarp;
    if (!take_all && !over) {
        // pack this CTA's bin-b0 keys for the cluster gather
        int nb0 = 0;
        for (int j = lane; j < ((wc + 31) & ~31); j += 32) {
            const bool hit = j < wc && (wkey[j] >> 21) == b0;
            nb0 += __popc(__ballot_sync(0xffffffffu, hit));
        }
        if (lane == 0) sh.wb0[warp] = nb0;
        __syncthreads();
        int off = 0;
        for (int w = 0; w < warp; ++w) off += sh.wb0[w];
        for (int j0 = 0; j0 < wc; j0 += 32) {
            const int j = j0 + lane;
            const bool hit = j < wc && (wkey[j] >> 21) == b0;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (hit) sh.cand[off + __popc(m & ((1u << lane) - 1u))] = wkey[j];
            off += __popc(m);
        }
        if (tid == 0) {
            int t = 0;
            for (int w = 0; w < kTopkWarps; ++w) t += sh.wb0[w];
            sh.ncand = t;
        }
    }
    if (tid == 0) sh.overflow = over;
    cluster.sync();   // lists, packed keys and flags complete; every CTA has read the row histogram
    if (EXT_HIST && rank == 0)
        for (int i = tid; i < kBins; i += kTopkThreads) a.ghist[(size_t)row * kBins + i] = 0u;
    int any_over = 0;
#pragma unroll
    for (int rr = 0; rr < kMaxCluster; ++rr) any_over |= rr < CS ? cluster.map_shared_rank(&sh, rr)->overflow : 0;

    // ---- 3. exact threshold theta and the ties at theta to take
    uint32_t theta = 0;
    int cnt[kMaxCluster];
    int ncand_all = 0;
#pragma unroll
    for (int rr = 0; rr < kMaxCluster; ++rr) {
        cnt[rr] = (rr < CS && !take_all && !any_over) ? cluster.map_shared_rank(&sh, rr)->ncand : 0;
        ncand_all += cnt[rr];
    }
    // the packed counts, not the histogram, decide: the gather can never overrun
    const bool local_ok = !take_all && !any_over && ncand_all <= kGatherCap;
    (void)in_b0;
    if (local_ok) {
        // flattened gather: a thread's remote loads are independent, in flight together
        int pre[kMaxCluster + 1];
        pre[0] = 0;
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) pre[rr + 1] = pre[rr] + cnt[rr];
        const int off = pre[kMaxCluster];
        constexpr int kG = kGatherCap / kTopkThreads;
        uint32_t v[kG];
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int i = u * kTopkThreads + tid;
            int rr = 0;
#pragma unroll
            for (int q = 1; q < kMaxCluster; ++q) rr += i >= pre[q];
            v[u] = i < off ? cluster.map_shared_rank(sh.cand, rr)[i - pre[rr]] : 0u;
        }
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int i = u * kTopkThreads + tid;
            if (i < off) sh.gathered[i] = v[u];
        }
        __syncthreads();
        uint32_t prefix = b0 << 21, pmask = 0xffe00000u;
        for (int pass = 1; pass < 3; ++pass) {
            const int shift = pass == 1 ? 10 : 0;
            const int nb = pass == 1 ? 2048 : 1024;
            for (int i = tid; i < nb; i += kTopkThreads) sh.hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < off; i += kTopkThreads) {
                const uint32_t k = sh.gathered[i];
                if ((k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & (uint32_t)(nb - 1)], 1u);
            }
            __syncthreads();
            find_bin(sh.hist, nb, krem, sh);
            prefix |= sh.bstar << shift;
            pmask |= (uint32_t)(nb - 1) << shift;
            krem -= sh.above;
            __syncthreads();
        }
        theta = prefix;
    }
    cluster.sync();   // remote reads of the packed keys are done
    if (!take_all && !local_ok) {
        // too many keys for shared memory: resolve the low 21 bits with
        // cluster-wide radix passes over the keys themselves
        uint32_t prefix = b0 << 21, pmask = 0xffe00000u;
        for (int pass = 1; pass < 3; ++pass) {
            const int shift = pass == 1 ? 10 : 0;
            const int nb = pass == 1 ? 2048 : 1024;
            for (int i = tid; i < nb; i += kTopkThreads) sh.hist[i] = 0;
            __syncthreads();
            for (int i0 = wbeg; i0 < wend; i0 += 128) {
                uint32_t k[4];
                load4(src, vec, i0 + lane * 4, wend, k);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (k[u] && (k[u] & pmask) == prefix) atomicAdd(&sh.hist[(k[u] >> shift) & (uint32_t)(nb - 1)], 1u);
            }
            cluster.sync();
            cluster_reduce(cluster, sh.hist, sh.red, nb, CS);
            cluster.sync();   // hist may be reset next pass only after every CTA has read it
            find_bin(sh.red, nb, krem, sh);
            prefix |= sh.bstar << shift;
            pmask |= (uint32_t)(nb - 1) << shift;
            krem -= sh.above;
            __syncthreads();
        }
        theta = prefix;
    }
    if (take_all) krem = 0;   // every valid key (key > 0 = theta) is taken

    // ---- 4. counts per warp (position order), offsets, compaction
    int gt = 0, eq = 0;
    if (!any_over) {
        for (int j = lane; j < wc; j += 32) {
            const uint32_t k = wkey[j];
            gt += k > theta;
            eq += k == theta;
        }
    } else {
        for (int i0 = wbeg; i0 < wend; i0 += 128) {
            uint32_t k[4];
            load4(src, vec, i0 + lane * 4, wend, k);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                gt += k[u] > theta;
                eq += k[u] == theta && i0 + lane * 4 + u < wend;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
        sh.warp_gt[warp] = gt;
        sh.warp_eq[warp] = eq;
    }
    __syncthreads();
    if (tid == 0) {
        int g = 0, e = 0;
        for (int w = 0; w < kTopkWarps; ++w) {
            g += sh.warp_gt[w];
            e += sh.warp_eq[w];
        }
        sh.cta_gt = g;
        sh.cta_eq = e;
    }
    cluster.sync();
    if (tid == 0) {
        // tie quota and output offset of every CTA, in rank (= position) order
        int cgt[kMaxCluster], ceq[kMaxCluster];
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) {
            const TopkShared* o = cluster.map_shared_rank(&sh, rr < CS ? rr : 0);
            cgt[rr] = rr < CS ? o->cta_gt : 0;
            ceq[rr] = rr < CS ? o->cta_eq : 0;
        }
        int eq_before = 0, sel_before = 0, eq_run = 0, sel_total = 0;
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) {
            int take = krem - eq_run;
            take = take < 0 ? 0 : (take > ceq[rr] ? ceq[rr] : take);
            if (rr == rank) {
                eq_before = eq_run;
                sel_before = sel_total;
            }
            eq_run += ceq[rr];
            sel_total += cgt[rr] + take;
        }
        int e = eq_before, s = sel_before;
        for (int w = 0; w < kTopkWarps; ++w) {
            sh.warp_eq_before[w] = e;
            sh.warp_sel_before[w] = s;
            int take = krem - e;
            take = take < 0 ? 0 : (take > sh.warp_eq[w] ? sh.warp_eq[w] : take);
            s += sh.warp_gt[w] + take;
            e += sh.warp_eq[w];
        }
        sh.total = sel_total;
    }
    __syncthreads();

    int32_t* out = a.idx + (size_t)row * a.B;
    const int32_t* bm = a.blkmap ? a.blkmap + (size_t)row * a.keep : nullptr;
    const int eq_before = sh.warp_eq_before[warp];
    int sel_pos = sh.warp_sel_before[warp];
    int eq_seen = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    auto emit = [&](bool in, uint32_t k, int c) {
        const bool is_eq = in && k == theta;
        const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
        const int rank_eq = eq_before + eq_seen + __popc(eqm & lt_mask);
        const bool take = in && (k > theta || (is_eq && rank_eq < krem));
        const unsigned sm = __ballot_sync(0xffffffffu, take);
        const int dst = sel_pos + __popc(sm & lt_mask);
        if (take && dst < a.B) {   // always true for a consistent histogram; never writes past B
            int pos = c;
            if (bm) {
                const int j = c / a.blk;
                pos = bm[j] * a.blk + (c - j * a.blk);
            }
            out[dst] = pos;
        }
        eq_seen += __popc(eqm);
        sel_pos += __popc(sm);
    };
    if (!any_over) {
        for (int j0 = 0; j0 < wc; j0 += 32) {
            const int j = j0 + lane;
            const bool in = j < wc;
            emit(in, in ? wkey[j] : 0u, in ? wpos[j] : 0);
        }
    } else {
        for (int i0 = wbeg; i0 < wend; i0 += 32) {
            const int i = i0 + lane;
            const bool in = i < wend;
            emit(in, in ? score_key(__ldcg(src + i)) : 0u, base + i);
        }
    }
    if (rank == CS - 1)
        for (int p = sh.total + tid; p < a.B; p += kTopkThreads) out[p] = -1;
    cluster.sync();   // keep this CTA's shared memory alive for remote readers
}

}  // namespace

cudaError_t launch_topk(const LaunchCtx& ctx, const float* scores, int rows, int n, int B, int32_t* idx,
                        const int32_t* blkmap, int blk, int keep, uint32_t* ghist) {
    TopkArgs a{};
    a.scores = scores;
    a.idx = idx;
    a.blkmap = blkmap;
    a.ghist = ghist;
    a.n = n;
    a.B = B;
    a.blk = blk;
    a.keep = keep;
    // Cluster size: about 16K keys per CTA, at most 8 (portable); fewer CTAs
    // per row when there are many rows.
    int cs = 1;
    while (cs < kMaxCluster && (long long)cs * 16384 < n) cs <<= 1;
    while (cs < kMaxCluster && (long long)rows * cs * 2 <= 2ll * ctx.num_sms && (long long)cs * 4096 < n) cs <<= 1;
    int seg = (n + cs - 1) / cs;
    seg = (seg + 127) & ~127;
    a.seg = seg;
    const size_t smem = sizeof(TopkShared);
    auto kern = ghist ? topk_cluster_kernel<true> : topk_cluster_kernel<false>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)cs, (unsigned)rows);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace lsa
