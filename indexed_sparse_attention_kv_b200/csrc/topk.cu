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
//   3. The keys of bin b0 of the whole cluster (in rank, hence position,
//      order) are gathered in every CTA; two local radix passes give the exact
//      threshold key theta and the number of ties at theta to take, and from
//      the same keys and the per-CTA list lengths every CTA derives its tie
//      quota and output offset: no further exchange.
//   4. Counts above / at theta per warp and a ballot compaction of the short
//      lists write the positions in ascending order.
// Whenever a list or the threshold bin is too large for shared memory (e.g.
// many equal scores), the cluster switches, uniformly, to radix passes and a
// compaction over the keys themselves, with the same result.
#include <cooperative_groups.h>

#include "block_select.cuh"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace cg = cooperative_groups;

namespace lsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins = 2048;
constexpr int kListPerWarp = 128;                       // (key, position) entries per warp
constexpr int kListCap = kListPerWarp * kTopkWarps;     // per CTA
constexpr int kGatherCap = 4096;                        // bin-b0 keys of the whole cluster
constexpr int kMaxCluster = 8;
constexpr int kBatch = 2;                               // 128-key steps whose loads are issued together

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
    uint32_t cand[kListCap];        // this CTA's bin-b0 keys (position order)
    uint32_t gathered[kGatherCap];  // the cluster's bin-b0 keys
    int wlist[kTopkWarps], wb0[kTopkWarps];
    int scan[kTopkWarps];
    int warp_gt[kTopkWarps], warp_eq[kTopkWarps];
    int warp_sel_before[kTopkWarps], warp_eq_before[kTopkWarps];
    int cta_gt, cta_eq, ncand, nlist, overflow;
    int rcnt[2 * kMaxCluster];      // per rank: gathered keys above / at theta
    uint32_t bstar;
    int above;
    int total;
};

// Given histogram `red` (nb bins) find the bin holding the krem-th largest
// element counted from the top; sets sh.bstar and sh.above (count above it)
// and returns the histogram total. All threads must call it.
__device__ __forceinline__ int find_bin(const uint32_t* red, int nb, int krem, TopkShared& sh) {
    const int per = nb / kTopkThreads;
    const int hi = nb - 1 - (int)threadIdx.x * per;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int local = 0;
    for (int q = 0; q < per; ++q) local += (int)red[hi - q];
    // two barriers: warp scans, warp totals through shared memory, then every
    // thread adds the totals of the warps above it
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sh.scan[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w) {
        const int t = sh.scan[w];
        before += w < warp ? t : 0;
        total += t;
    }
    const int above_me = before + incl - local;
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

// kBatch 128-key steps of a warp range starting at i00 (lane: 4 consecutive
// keys per step): every load is issued before any key is converted, so a
// thread's loads are all in flight together.
__device__ __forceinline__ void load_batch(const float* src, bool vec, int i00, int end, int lane,
                                           uint32_t (&kk)[kBatch][4]) {
    if (vec && i00 + 128 * kBatch <= end) {
        float4 v[kBatch];
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub)
            v[ub] = __ldcg(reinterpret_cast<const float4*>(src + i00 + ub * 128 + lane * 4));
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) {
            kk[ub][0] = score_key(v[ub].x);
            kk[ub][1] = score_key(v[ub].y);
            kk[ub][2] = score_key(v[ub].z);
            kk[ub][3] = score_key(v[ub].w);
        }
    } else {
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) load4(src, vec, i00 + ub * 128 + lane * 4, end, kk[ub]);
    }
}

// As load_batch, the raw scores (NaN past `end`): the list pass compares them
// with a float threshold and converts only its hits to order keys.
__device__ __forceinline__ void load_batch_f(const float* src, bool vec, int i00, int end, int lane,
                                             float (&ff)[kBatch][4]) {
    if (vec && i00 + 128 * kBatch <= end) {
        float4 v[kBatch];
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub)
            v[ub] = __ldcg(reinterpret_cast<const float4*>(src + i00 + ub * 128 + lane * 4));
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) {
            ff[ub][0] = v[ub].x;
            ff[ub][1] = v[ub].y;
            ff[ub][2] = v[ub].z;
            ff[ub][3] = v[ub].w;
        }
    } else {
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i00 + ub * 128 + lane * 4 + u;
                ff[ub][u] = i < end ? __ldcg(src + i) : __int_as_float(0x7fc00000);
            }
    }
}

template <bool EXT_HIST>
__global__ void __launch_bounds__(kTopkThreads, 2) topk_cluster_kernel(const TopkArgs a) {
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
            load_batch(src, vec, i00, wend, lane, kk);
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
    // Coalesced steps of 128 keys (lane: 4 consecutive keys, one 16-byte load;
    // every load of a batch issued before any use); four ballots per step give
    // each hit its rank in position order without a shuffle scan. A score is
    // in bin >= b0 iff it is >= the smallest float of bin b0 (NaN: never), so
    // only the hits are converted to order keys.
    uint32_t* wkey = sh.lkey + warp * kListPerWarp;
    int* wpos = sh.lpos + warp * kListPerWarp;
    int wc = 0;
    const unsigned lt = (1u << lane) - 1u;
    const float thr_b0 = key_floor(b0 << 21);
    for (int i00 = wbeg; i00 < wend; i00 += 128 * kBatch) {
        float ff[kBatch][4];
        load_batch_f(src, vec, i00, wend, lane, ff);
#pragma unroll
        for (int ub = 0; ub < kBatch; ++ub) {
            unsigned m[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) m[u] = __ballot_sync(0xffffffffu, ff[ub][u] >= thr_b0);
            int slot = wc + __popc(m[0] & lt) + __popc(m[1] & lt) + __popc(m[2] & lt) + __popc(m[3] & lt);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if ((m[u] >> lane) & 1u) {
                    if (slot < kListPerWarp) {
                        wkey[slot] = score_key(ff[ub][u]);
                        wpos[slot] = base + i00 + ub * 128 + lane * 4 + u;
                    }
                    ++slot;
                }
            }
            wc += __popc(m[0]) + __popc(m[1]) + __popc(m[2]) + __popc(m[3]);
        }
    }
    if (lane == 0) sh.wlist[warp] = wc;
    __syncthreads();
    bool over = false;
    for (int w = 0; w < kTopkWarps; ++w) over |= sh.wlist[w] > kListPerWarp;
    if (!take_all && !over) {
        // pack this CTA's bin-b0 keys (position order) for the cluster gather
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
    }
    if (tid == 0) {
        int nl = 0, nc = 0;
        for (int w = 0; w < kTopkWarps; ++w) {
            nl += sh.wlist[w];
            nc += (!take_all && !over) ? sh.wb0[w] : 0;
        }
        sh.nlist = nl;
        sh.ncand = nc;
        sh.overflow = over;
    }
    cluster.sync();   // lists, packed keys and counts complete; every CTA has read the row histogram
    if (EXT_HIST && rank == 0)
        for (int i = tid; i < kBins; i += kTopkThreads) a.ghist[(size_t)row * kBins + i] = 0u;
    int any_over = 0, cnt[kMaxCluster], nl[kMaxCluster];
#pragma unroll
    for (int rr = 0; rr < kMaxCluster; ++rr) {
        const TopkShared* o = cluster.map_shared_rank(&sh, rr < CS ? rr : 0);
        any_over |= rr < CS ? o->overflow : 0;
        cnt[rr] = rr < CS ? o->ncand : 0;
        nl[rr] = rr < CS ? o->nlist : 0;
    }
    int pre[kMaxCluster + 1];
    pre[0] = 0;
#pragma unroll
    for (int rr = 0; rr < kMaxCluster; ++rr) pre[rr + 1] = pre[rr] + cnt[rr];
    const int ncand_all = pre[kMaxCluster];
    (void)in_b0;
    // uniform over the cluster: every CTA read the same counts
    const bool fast = !any_over && (take_all || ncand_all <= kGatherCap);

    int32_t* out = a.idx + (size_t)row * a.B;
    const int32_t* bm = a.blkmap ? a.blkmap + (size_t)row * a.keep : nullptr;
    const unsigned lt_mask = (1u << lane) - 1u;
    uint32_t theta = 0;
    int eq_before = 0, sel_pos = 0, eq_seen = 0;
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
    // per-warp counts of keys above / at theta, reduced into sh.warp_gt / warp_eq
    auto warp_counts = [&](int gt, int eq) {
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
    };
    // warp offsets from this CTA's tie base and output base (thread 0)
    auto warp_offsets = [&](int e, int s_) {
        for (int w = 0; w < kTopkWarps; ++w) {
            sh.warp_eq_before[w] = e;
            sh.warp_sel_before[w] = s_;
            int take = krem - e;
            take = take < 0 ? 0 : (take > sh.warp_eq[w] ? sh.warp_eq[w] : take);
            s_ += sh.warp_gt[w] + take;
            e += sh.warp_eq[w];
        }
    };

    if (fast) {
        // ---- 3. theta from the cluster's bin-b0 keys, gathered into every CTA
        int eq_rank = 0, sel_rank = 0, sel_total = 0;
        if (!take_all) {
            constexpr int kG = kGatherCap / kTopkThreads;
            uint32_t v[kG];
#pragma unroll
            for (int u = 0; u < kG; ++u) {
                const int i = u * kTopkThreads + tid;
                int rr = 0;
#pragma unroll
                for (int q = 1; q < kMaxCluster; ++q) rr += i >= pre[q];
                v[u] = i < ncand_all ? cluster.map_shared_rank(sh.cand, rr)[i - pre[rr]] : 0u;
            }
#pragma unroll
            for (int u = 0; u < kG; ++u) {
                const int i = u * kTopkThreads + tid;
                if (i < ncand_all) sh.gathered[i] = v[u];
            }
            // both local histograms (bits 10..20 in hist, bits 0..9 in red, whose
            // row histogram is no longer needed) are cleared up front
            for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[i] = 0;
            for (int i = tid; i < 1024; i += kTopkThreads) sh.red[i] = 0;
            if (tid < 2 * kMaxCluster) sh.rcnt[tid] = 0;
            __syncthreads();
            uint32_t prefix = b0 << 21;
            for (int i = tid; i < ncand_all; i += kTopkThreads)
                atomicAdd(&sh.hist[(sh.gathered[i] >> 10) & 2047u], 1u);
            __syncthreads();
            find_bin(sh.hist, 2048, krem, sh);
            prefix |= sh.bstar << 10;
            krem -= sh.above;
            for (int i = tid; i < ncand_all; i += kTopkThreads) {
                const uint32_t k = sh.gathered[i];
                if ((k & 0xfffffc00u) == prefix) atomicAdd(&sh.red[k & 1023u], 1u);
            }
            __syncthreads();
            find_bin(sh.red, 1024, krem, sh);
            prefix |= sh.bstar;
            krem -= sh.above;
            theta = prefix;
            // per-rank counts above / at theta among the gathered keys (rank ranges)
            for (int i = tid; i < ncand_all; i += kTopkThreads) {
                int rr = 0;
#pragma unroll
                for (int q = 1; q < kMaxCluster; ++q) rr += i >= pre[q];
                const uint32_t k = sh.gathered[i];
                if (k > theta) atomicAdd(&sh.rcnt[rr], 1);
                else if (k == theta) atomicAdd(&sh.rcnt[kMaxCluster + rr], 1);
            }
            __syncthreads();
            int eq_run = 0, sel_run = 0;
#pragma unroll
            for (int rr = 0; rr < kMaxCluster; ++rr) {
                if (rr < CS) {
                    const int req = sh.rcnt[kMaxCluster + rr];
                    int take = krem - eq_run;
                    take = take < 0 ? 0 : (take > req ? req : take);
                    if (rr == rank) {
                        eq_rank = eq_run;
                        sel_rank = sel_run;
                    }
                    eq_run += req;
                    sel_run += (nl[rr] - cnt[rr]) + sh.rcnt[rr] + take;
                }
            }
            sel_total = sel_run;
        } else {
            krem = 0;   // every valid key (key > 0 = theta) is taken
            int sel_run = 0;
#pragma unroll
            for (int rr = 0; rr < kMaxCluster; ++rr) {
                if (rr == rank) sel_rank = sel_run;
                sel_run += nl[rr];   // zero for rr >= CS
            }
            sel_total = sel_run;
        }
        // ---- 4. counts over this warp's list, offsets, compaction of the list
        int gt = 0, eq = 0;
        for (int j = lane; j < wc; j += 32) {
            const uint32_t k = wkey[j];
            gt += k > theta;
            eq += k == theta;
        }
        warp_counts(gt, eq);
        if (tid == 0) {
            warp_offsets(eq_rank, sel_rank);
            sh.total = sel_total;
        }
        __syncthreads();
        eq_before = sh.warp_eq_before[warp];
        sel_pos = sh.warp_sel_before[warp];
        for (int j0 = 0; j0 < wc; j0 += 32) {
            const int j = j0 + lane;
            const bool in = j < wc;
            emit(in, in ? wkey[j] : 0u, in ? wpos[j] : 0);
        }
    } else {
        // ---- 3'. too many keys for shared memory: resolve the low 21 bits with
        // cluster-wide radix passes over the keys themselves
        if (!take_all) {
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
                        if (k[u] && (k[u] & pmask) == prefix)
                            atomicAdd(&sh.hist[(k[u] >> shift) & (uint32_t)(nb - 1)], 1u);
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
        } else {
            krem = 0;
        }
        // ---- 4'. counts over the keys, cluster exchange, compaction of the keys
        int gt = 0, eq = 0;
        for (int i0 = wbeg; i0 < wend; i0 += 128) {
            uint32_t k[4];
            load4(src, vec, i0 + lane * 4, wend, k);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                gt += k[u] > theta;
                eq += k[u] == theta && i0 + lane * 4 + u < wend;
            }
        }
        warp_counts(gt, eq);
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
            int e0 = 0, s0 = 0, eq_run = 0, sel_total = 0;
#pragma unroll
            for (int rr = 0; rr < kMaxCluster; ++rr) {
                int take = krem - eq_run;
                take = take < 0 ? 0 : (take > ceq[rr] ? ceq[rr] : take);
                if (rr == rank) {
                    e0 = eq_run;
                    s0 = sel_total;
                }
                eq_run += ceq[rr];
                sel_total += cgt[rr] + take;
            }
            warp_offsets(e0, s0);
            sh.total = sel_total;
        }
        __syncthreads();
        eq_before = sh.warp_eq_before[warp];
        sel_pos = sh.warp_sel_before[warp];
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

// Rows of at most NT * ITEMS keys: one CTA per row holds the whole row in
// registers (ITEMS per thread) and runs the exact block selection (radix
// passes on the order keys, boundary ties to the lower position, ascending
// output through a bitmap). Positions of coarse-to-fine candidates map
// through blkmap. ITEMS is the smallest of 4 and 16 that holds the row, so
// short rows do not loop over empty registers in every pass.
constexpr int kSmallItems = 16;

template <int NT, int ITEMS>
__global__ void __launch_bounds__(NT) topk_small_kernel(const TopkArgs a) {
    __shared__ BlockSelShared sh;
    extern __shared__ uint32_t sbitmap[];
    const int row = blockIdx.x;
    const float* src = a.scores + (size_t)row * a.n;
    pdl_launch_dependents();
    pdl_wait();   // the scores come from the previous kernel
    uint32_t kk[ITEMS];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int i = (int)threadIdx.x + it * NT;
        kk[it] = i < a.n ? score_key(__ldcg(src + i)) : 0u;
    }
    if (a.ghist)   // the scorer's histogram is not needed here; leave it zero for the next step
        for (int i = threadIdx.x; i < kBins; i += NT) a.ghist[(size_t)row * kBins + i] = 0u;
    const int32_t* bm = a.blkmap ? a.blkmap + (size_t)row * a.keep : nullptr;
    select_and_emit<NT>(
        [&](auto f) {
#pragma unroll
            for (int it = 0; it < ITEMS; ++it)
                if (kk[it]) f(kk[it], (uint32_t)((int)threadIdx.x + it * NT));
        },
        a.B, a.n, sh, sbitmap, a.idx + (size_t)row * a.B,
        a.B, [&](int i) -> int32_t { return bm ? bm[i / a.blk] * a.blk + i % a.blk : i; });
}

template <int NT, int ITEMS>
cudaError_t launch_small(const LaunchCtx& ctx, const TopkArgs& a, int rows) {
    const int smem = (a.n + 31) / 32 * 4;
    auto kern = topk_small_kernel<NT, ITEMS>;
    cudaError_t e = ensure_dyn_smem((const void*)kern, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];   // prologue overlaps the previous kernel's tail
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
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
    // rows of up to 4K keys, and up to 16K keys unless the set is short: one
    // 1024-thread CTA per row (measured faster than 256 or 512 threads for
    // 4K-key rows: the selection's passes and barriers, not the loads, set
    // its time). A short set from a longer row (B <= n / 16, as the coarse
    // stage's kept blocks) goes to the cluster instead, whose CTAs share the
    // row while its lists stay short.
    if (n <= 1024 * 4) return launch_small<1024, 4>(ctx, a, rows);
    if (n <= 1024 * kSmallItems && (long long)B * 16 > n) return launch_small<1024, kSmallItems>(ctx, a, rows);
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
    // Launched without programmatic dependent launch: placing 8-CTA clusters
    // while the scorer's CTAs drain fragments the GPCs and pushed the last
    // clusters into a second wave (measured); a plain launch places them all.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace lsa
