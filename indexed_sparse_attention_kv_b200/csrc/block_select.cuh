// Exact block-wide top-B selection shared by the top-B kernels: radix
// selection of the B-th largest order key over the items a CTA holds, ties at
// the boundary resolved toward the lower item index, and emission of the
// selected items in ascending item order through a bitmap.
#pragma once

#include <stdint.h>

#include "lsa_common.cuh"

namespace lsa {

constexpr int kEqList = 1024;         // boundary ties resolved by direct ranking up to this many

struct BlockSelShared {
    uint32_t hist[2048];
    int wtot[32];
    int bin, above, eqc;
    int neq;
    uint32_t pos_thr;
    uint32_t eqpos[kEqList];
};

// Exclusive block-wide prefix sum of v (thread order); *total = the sum.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* wtot, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wtot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = lane < NT / 32 ? wtot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NT / 32) wtot[lane] = w;
    }
    __syncthreads();
    const int before = wid ? wtot[wid - 1] : 0;
    *total = wtot[NT / 32 - 1];
    __syncthreads();
    return before + x - v;
}

// Block-wide radix selection (11 + 11 + 10 bits) of the need-th largest
// non-zero key. `visit(f)` calls f(key, position) for every item this thread
// holds (key 0 = no item). Results, identical in every thread: *theta = that
// key, *n_gt = keys above it, *n_eq = keys equal to it, *total = non-zero
// keys. With fewer than `need` keys: theta = 0, n_gt = total.
template <int NT, class V>
__device__ void block_select(V visit, int need, BlockSelShared& sh, uint32_t* theta, int* n_gt, int* n_eq, int* total) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0, pmask = 0;
    int rem = need, gt = 0, eqc = 0;
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < 2048; i += NT) sh.hist[i] = 0;
        __syncthreads();
        visit([&](uint32_t k, uint32_t) {
            if (k != 0u && (k & pmask) == prefix) atomicAdd(&sh.hist[(k >> shift) & (uint32_t)(nb - 1)], 1u);
        });
        __syncthreads();
        const int per = nb / NT;
        const int top = nb - 1 - tid * per;
        int s = 0;
        for (int j = 0; j < per; ++j) s += (int)sh.hist[top - j];
        int tot = 0;
        const int excl = block_excl_scan<NT>(s, sh.wtot, &tot);
        if (pass == 0) {
            *total = tot;
            if (tot < need) {
                *theta = 0u;
                *n_gt = tot;
                *n_eq = 0;
                return;
            }
        }
        if (excl < rem && rem <= excl + s) {
            int c = excl;
            for (int j = 0; j < per; ++j) {
                const int b = top - j;
                const int hb = (int)sh.hist[b];
                if (c + hb >= rem) {
                    sh.bin = b;
                    sh.above = c;
                    sh.eqc = hb;
                    break;
                }
                c += hb;
            }
        }
        __syncthreads();
        const int b = sh.bin;
        rem -= sh.above;
        gt += sh.above;
        eqc = sh.eqc;
        prefix |= (uint32_t)b << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    *theta = prefix;
    *n_gt = gt;
    *n_eq = eqc;
}

// The top `need` items of `visit` (keys desc, ties: lower item index), written
// in ascending item order as pos_of(item) to out[0 .. need), out[need .. B)
// = -1. bitmap: 4 * ceil(n / 32) bytes of shared memory; items are < n.
template <int NT, class V, class M>
__device__ __forceinline__ void select_and_emit(V visit, int need, int n, BlockSelShared& sh, uint32_t* bitmap,
                                                int32_t* out, int B, M pos_of) {
    if (threadIdx.x == 0) sh.neq = 0;   // visible after block_select's barriers
    uint32_t theta;
    int gt, eq, total;
    block_select<NT>(visit, need, sh, &theta, &gt, &eq, &total);
    uint32_t pos_thr = 0xFFFFFFFFu;
    const int need_eq = need - gt;
    if (theta != 0u && eq > need_eq) {
        // Equal keys at the boundary: keep the need_eq lowest positions.
        if (eq <= kEqList) {
            visit([&](uint32_t k, uint32_t pos) {
                if (k == theta) sh.eqpos[atomicAdd(&sh.neq, 1)] = pos;
            });
            __syncthreads();
            for (int i = threadIdx.x; i < eq; i += NT) {
                const uint32_t mine = sh.eqpos[i];
                int rank = 0;
                for (int j = 0; j < eq; ++j) rank += sh.eqpos[j] < mine ? 1 : 0;
                if (rank == need_eq - 1) sh.pos_thr = mine;
            }
            __syncthreads();
            pos_thr = sh.pos_thr;
        } else {
            uint32_t th2;
            int g2, e2, t2;
            block_select<NT>(
                [&](auto f) { visit([&](uint32_t k, uint32_t pos) { f(k == theta ? ~pos : 0u, pos); }); }, need_eq,
                sh, &th2, &g2, &e2, &t2);
            pos_thr = ~th2;
        }
    }
    const int nw = (n + 31) >> 5;
    for (int w = threadIdx.x; w < nw; w += NT) bitmap[w] = 0u;
    __syncthreads();
    visit([&](uint32_t k, uint32_t pos) {
        if (k != 0u && (k > theta || (k == theta && pos <= pos_thr))) atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
    });
    __syncthreads();
    const int per = (nw + NT - 1) / NT;
    const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bitmap[w]);
    int nsel = 0;
    int o = block_excl_scan<NT>(c, sh.wtot, &nsel);
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (o < B) out[o] = pos_of(w * 32 + b);
            ++o;
        }
    }
    for (int j = nsel + threadIdx.x; j < B; j += NT) out[j] = -1;
}

}  // namespace lsa
