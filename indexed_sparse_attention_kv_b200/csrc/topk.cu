// Deterministic top-B selection per row with a thread-block-cluster radix select.
//
// Joint Subspace Sparse Attention for Efficient Long-Context Decoding, Fig. 1:
// each KV head keeps the B token positions with the largest scores. Ties at
// the threshold go to the lower position; the set is written in ascending order
// and padded with -1 when fewer than B candidates (non-NaN scores) exist.
//
// One cluster of CS CTAs owns a row; CTA k owns a contiguous segment of it.
// Scores map to order-preserving 32-bit keys (NaN -> 0, never selected).
//   1. histogram of the top 11 key bits (warp-aggregated shared atomics);
//      every CTA sums the cluster's histograms through distributed shared
//      memory and finds the bin b0 that holds the B-th largest key;
//   2. every CTA collects its keys that fall in b0; when the cluster holds few
//      of them, every CTA gathers all of them and resolves the exact threshold
//      key theta (and how many ties at theta to take) with two local radix
//      passes; otherwise two more cluster-wide radix passes do it;
//   3. per-warp counts of keys above / equal to theta, exclusive prefix sums
//      over warps and over the cluster's CTAs, and a compaction pass with warp
//      ballots in position order write the selected positions ascending.
#include <cooperative_groups.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace cg = cooperative_groups;

namespace lsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kSegCap = 16384;     // keys staged in shared memory per CTA (64 KiB)
constexpr int kBins = 2048;
constexpr int kCandCap = 4096;     // threshold-bin keys kept per CTA
constexpr int kGatherCap = 4096;   // threshold-bin keys gathered from the whole cluster
constexpr int kMaxCluster = 8;

struct TopkArgs {
    const float* scores;      // [rows, n]
    int32_t* idx;             // [rows, B]
    const int32_t* blkmap;    // optional [rows, keep]: candidate c -> blkmap[c / blk] * blk + c % blk
    int n, B, seg, staged, blk, keep;
};

struct TopkShared {
    union {
        struct {
            uint32_t hist[kBins];
            uint32_t red[kBins];
        } h;
        uint32_t gathered[kGatherCap];
    } u;
    uint32_t lhist[kBins];
    uint32_t cand[kCandCap];
    int scan[kTopkWarps];
    int warp_gt[kTopkWarps], warp_eq[kTopkWarps];
    int warp_sel_before[kTopkWarps], warp_eq_before[kTopkWarps];
    int cta_gt, cta_eq, ncand;
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

// Warp-aggregated histogram increment: lanes with equal bins add once.
__device__ __forceinline__ void hist_add(uint32_t* h, bool active, uint32_t bin) {
    const uint32_t key = active ? bin : 0xffffffffu;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(peers) - 1;
    if (active && (int)(threadIdx.x & 31) == leader) atomicAdd(&h[bin], (uint32_t)__popc(peers));
}

// Sum histogram `h` (nb bins) over the cluster's CTAs into `red`.
__device__ __forceinline__ void cluster_reduce(cg::cluster_group& cluster, uint32_t* h, uint32_t* red, int nb, int CS) {
    for (int bin = threadIdx.x; bin < nb; bin += kTopkThreads) {
        uint32_t v[kMaxCluster];
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) v[rr] = rr < CS ? cluster.map_shared_rank(h, rr)[bin] : 0u;
        uint32_t s = 0;
#pragma unroll
        for (int rr = 0; rr < kMaxCluster; ++rr) s += v[rr];
        red[bin] = s;
    }
}

__global__ void __launch_bounds__(kTopkThreads) topk_cluster_kernel(const TopkArgs a) {
    cg::cluster_group cluster = cg::this_cluster();
    const int CS = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    __shared__ TopkShared sh;
    extern __shared__ uint32_t keys[];

    const int base = rank * a.seg;
    int len = a.n - base;
    len = len < 0 ? 0 : (len > a.seg ? a.seg : len);
    const float* src = a.scores + (size_t)row * a.n + base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (a.staged)
        for (int i = tid; i < len; i += kTopkThreads) keys[i] = score_key(src[i]);
    auto key_at = [&](int i) -> uint32_t { return a.staged ? keys[i] : score_key(src[i]); };
    const int len_up = (len + 31) & ~31;

    // ---- 1. top-11-bit histogram, cluster sum, threshold bin b0
    for (int i = tid; i < kBins; i += kTopkThreads) sh.u.h.hist[i] = 0;
    if (tid == 0) sh.ncand = 0;
    __syncthreads();
    for (int i = tid; i < len_up; i += kTopkThreads) {
        const uint32_t k = i < len ? key_at(i) : 0u;
        hist_add(sh.u.h.hist, k != 0u, k >> 21);
    }
    cluster.sync();
    cluster_reduce(cluster, sh.u.h.hist, sh.u.h.red, kBins, CS);
    __syncthreads();
    int krem = a.B;
    const int total = find_bin(sh.u.h.red, kBins, krem, sh);
    const bool take_all = total <= a.B;
    uint32_t theta = 0;
    if (!take_all) {
        const uint32_t b0 = sh.bstar;
        krem -= sh.above;
        const int in_b0 = (int)sh.u.h.red[b0];
        // ---- 2. collect this CTA's keys in b0
        for (int i = tid; i < len_up; i += kTopkThreads) {
            const uint32_t k = i < len ? key_at(i) : 0u;
            const bool hit = k != 0u && (k >> 21) == b0;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            int off = 0;
            if (lane == 0 && m) off = atomicAdd(&sh.ncand, __popc(m));
            off = __shfl_sync(0xffffffffu, off, 0);
            const int slot = off + __popc(m & ((1u << lane) - 1u));
            if (hit && slot < kCandCap) sh.cand[slot] = k;
        }
        cluster.sync();   // every CTA's hist/red reads are done; candidate lists complete
        const bool local_ok = in_b0 <= kGatherCap;
        if (local_ok) {
            // gather the cluster's b0 keys (rank order), then two local radix passes
            int off = 0;
            for (int rr = 0; rr < CS; ++rr) {
                const TopkShared* o = cluster.map_shared_rank(&sh, rr);
                const int nc = min(o->ncand, kCandCap);
                for (int i = tid; i < nc; i += kTopkThreads) sh.u.gathered[off + i] = o->cand[i];
                off += nc;
            }
            __syncthreads();
            uint32_t prefix = b0 << 21, pmask = 0xffe00000u;
            for (int pass = 1; pass < 3; ++pass) {
                const int shift = pass == 1 ? 10 : 0;
                const int nb = pass == 1 ? 2048 : 1024;
                for (int i = tid; i < nb; i += kTopkThreads) sh.lhist[i] = 0;
                __syncthreads();
                for (int i = tid; i < ((off + 31) & ~31); i += kTopkThreads) {
                    const uint32_t k = i < off ? sh.u.gathered[i] : 0u;
                    hist_add(sh.lhist, i < off && (k & pmask) == prefix, (k >> shift) & (uint32_t)(nb - 1));
                }
                __syncthreads();
                find_bin(sh.lhist, nb, krem, sh);
                prefix |= sh.bstar << shift;
                pmask |= (uint32_t)(nb - 1) << shift;
                krem -= sh.above;
                __syncthreads();
            }
            theta = prefix;
        }
        cluster.sync();   // remote readers of cand / ncand are done
        if (!local_ok) {
            // many keys share b0: resolve the low 21 bits with cluster-wide passes
            uint32_t prefix = b0 << 21, pmask = 0xffe00000u;
            for (int pass = 1; pass < 3; ++pass) {
                const int shift = pass == 1 ? 10 : 0;
                const int nb = pass == 1 ? 2048 : 1024;
                uint32_t* h = sh.lhist;
                for (int i = tid; i < nb; i += kTopkThreads) h[i] = 0;
                __syncthreads();
                for (int i = tid; i < len_up; i += kTopkThreads) {
                    const uint32_t k = i < len ? key_at(i) : 0u;
                    hist_add(h, k != 0u && (k & pmask) == prefix, (k >> shift) & (uint32_t)(nb - 1));
                }
                cluster.sync();
                cluster_reduce(cluster, h, sh.u.h.red, nb, CS);
                cluster.sync();   // lhist may be reset next pass only after every CTA has read it
                find_bin(sh.u.h.red, nb, krem, sh);
                prefix |= sh.bstar << shift;
                pmask |= (uint32_t)(nb - 1) << shift;
                krem -= sh.above;
                __syncthreads();
            }
            theta = prefix;
        }
    } else {
        krem = 0;   // every candidate (key > 0) is selected
    }

    // ---- 3. counts per warp over contiguous warp ranges (position order)
    int wlen = (len + kTopkWarps - 1) / kTopkWarps;
    wlen = (wlen + 31) & ~31;
    const int wbeg = min(len, warp * wlen), wend = min(len, wbeg + wlen);
    int gt = 0, eq = 0;
    for (int i = wbeg + lane; i < wend; i += 32) {
        const uint32_t k = key_at(i);
        gt += k > theta;
        eq += k == theta;
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
        // Tie quota and output offset of every CTA, in rank (= position) order.
        int eq_before = 0, sel_before = 0, eq_run = 0, sel_total = 0;
        for (int rr = 0; rr < CS; ++rr) {
            const TopkShared* o = cluster.map_shared_rank(&sh, rr);
            int take = krem - eq_run;
            take = take < 0 ? 0 : (take > o->cta_eq ? o->cta_eq : take);
            if (rr == rank) {
                eq_before = eq_run;
                sel_before = sel_total;
            }
            eq_run += o->cta_eq;
            sel_total += o->cta_gt + take;
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

    // ---- compaction in position order
    int32_t* out = a.idx + (size_t)row * a.B;
    const int32_t* bm = a.blkmap ? a.blkmap + (size_t)row * a.keep : nullptr;
    const int eq_before = sh.warp_eq_before[warp];
    int sel_pos = sh.warp_sel_before[warp];
    int eq_seen = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i0 = wbeg; i0 < wend; i0 += 32) {
        const int i = i0 + lane;
        const bool in = i < wend;
        const uint32_t k = in ? key_at(i) : 0u;
        const bool is_eq = in && k == theta;
        const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
        const int rank_eq = eq_before + eq_seen + __popc(eqm & lt_mask);
        const bool take = in && (k > theta || (is_eq && rank_eq < krem));
        const unsigned sm = __ballot_sync(0xffffffffu, take);
        if (take) {
            const int c = base + i;
            int pos = c;
            if (bm) {
                const int j = c / a.blk;
                pos = bm[j] * a.blk + (c - j * a.blk);
            }
            out[sel_pos + __popc(sm & lt_mask)] = pos;
        }
        eq_seen += __popc(eqm);
        sel_pos += __popc(sm);
    }
    if (rank == CS - 1)
        for (int p = sh.total + tid; p < a.B; p += kTopkThreads) out[p] = -1;
    cluster.sync();   // keep this CTA's shared memory alive for remote readers
}

}  // namespace

cudaError_t launch_topk(const LaunchCtx& ctx, const float* scores, int rows, int n, int B, int32_t* idx,
                        const int32_t* blkmap, int blk, int keep) {
    TopkArgs a{};
    a.scores = scores;
    a.idx = idx;
    a.blkmap = blkmap;
    a.n = n;
    a.B = B;
    a.blk = blk;
    a.keep = keep;
    // Cluster size: enough CTAs to spread the row, at most 8 (portable).
    int cs = 1;
    while (cs < kMaxCluster && (long long)cs * 4096 < n) cs <<= 1;
    // Prefer fewer CTAs per row when there are many rows.
    while (cs > 1 && (long long)rows * cs > 4ll * ctx.num_sms && (n + cs / 2 - 1) / (cs / 2) <= kSegCap) cs >>= 1;
    int seg = (n + cs - 1) / cs;
    seg = (seg + 31) & ~31;
    a.seg = seg;
    a.staged = seg <= kSegCap;
    const size_t dyn = a.staged ? (size_t)seg * 4 : 0;
    cudaError_t e = ensure_dyn_smem((const void*)topk_cluster_kernel, (int)(kSegCap * 4));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)cs, (unsigned)rows);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace lsa
