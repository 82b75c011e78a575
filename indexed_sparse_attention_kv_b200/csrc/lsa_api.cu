// C-ABI layer of liblsa.so: argument validation, workspace layout and launch
// sequencing on the caller's stream. Declarations and contracts: include/lsa.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/lsa.h"
#include "lsa_internal.h"

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;       // device status word + reserved
constexpr long long kDefaultWaitLimit = 2000000000ll;   // ns of device time

std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

int device_sms() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cache[dev].load() > 0) return cache[dev].load();
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev >= 0 && dev < 64) cache[dev].store(n);
    return n;
}

lsa::LaunchCtx make_ctx(void* stream) {
    lsa::LaunchCtx c;
    c.stream = reinterpret_cast<cudaStream_t>(stream);
    c.num_sms = device_sms();
    c.wait_limit = g_wait_limit.load();
    return c;
}

lsa_status check_dims(const lsa_dims* d) {
    if (!d) return LSA_ERR_ARG;
    if (d->batch < 1 || d->hq < 1 || d->hkv < 1 || d->d < 1 || d->r < 1 || d->T < 1) return LSA_ERR_ARG;
    if (d->hq % d->hkv != 0) return LSA_ERR_ARG;
    const int G = d->hq / d->hkv;
    if (!pow2_in(G, 1, 16)) return LSA_ERR_UNSUPPORTED;
    if (!(d->r == 16 || d->r == 32 || d->r == 64 || d->r == 128)) return LSA_ERR_UNSUPPORTED;
    if (!(d->d == 64 || d->d == 128 || d->d == 256)) return LSA_ERR_UNSUPPORTED;
    if ((long long)d->hkv * d->r > 4096) return LSA_ERR_UNSUPPORTED;
    return LSA_OK;
}

lsa_status check_B(int B) {
    if (B < 1) return LSA_ERR_ARG;
    if (B > 65536) return LSA_ERR_UNSUPPORTED;
    return LSA_OK;
}

// The attention entries only read index sets, so they accept longer ones (an
// index set may cover a whole 128K cache: the dense full-KV comparison).
constexpr int kMaxAttnB = 1 << 24;
lsa_status check_B_attn(int B) {
    if (B < 1) return LSA_ERR_ARG;
    if (B > kMaxAttnB) return LSA_ERR_UNSUPPORTED;
    return LSA_OK;
}

lsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA; }

// Workspace layout (byte offsets from the 256-byte aligned base).
struct DecodeLayout {
    size_t status = 0;        // uint32 device status word
    size_t scores = 0;        // fp32 [batch, hkv, T]   (flat) or coarse [batch, hkv, nblk]
    size_t fine = 0;          // fp32 [batch, hkv, keep * blk]  (hierarchical)
    size_t blkidx = 0;        // int32 [batch, hkv, keep]       (hierarchical)
    size_t idx = 0;           // int32 [batch, hkv, B]
    size_t pm = 0, pl = 0, po = 0;
    size_t counters = 0;      // uint32 [batch, hkv] attention segment counters
    size_t hist = 0;          // uint32 [batch, hkv, 2048] order-key histogram (scorer -> top-B)
    size_t total = 0;
    lsa::AttnPlan plan{};
};

DecodeLayout decode_layout(const lsa_dims* d, int B, int blk, int keep, int num_sms) {
    DecodeLayout L;
    size_t off = kHeaderBytes;
    const size_t units = (size_t)d->batch * d->hkv;
    const size_t nscore = blk > 0 ? (size_t)(d->T + blk - 1) / blk : (size_t)d->T;
    L.scores = off;
    off = align_up(off + units * nscore * 4);
    if (blk > 0) {
        L.fine = off;
        off = align_up(off + units * (size_t)keep * blk * 4);
        L.blkidx = off;
        off = align_up(off + units * (size_t)keep * 4);
    }
    L.idx = off;
    off = align_up(off + units * (size_t)B * 4);
    const int G = d->hq / d->hkv;
    L.plan = lsa::plan_attn(d->batch, d->hkv, G, B, d->d, num_sms);
    const size_t slots = units * (size_t)L.plan.smax * G;
    L.pm = off;
    off = align_up(off + slots * 4);
    L.pl = off;
    off = align_up(off + slots * 4);
    L.po = off;
    off = align_up(off + slots * (size_t)d->d * 4);
    L.counters = off;
    off = align_up(off + units * 4);
    L.hist = off;
    off = align_up(off + units * 2048 * 4);
    L.total = off;
    return L;
}

// Prefill workspace: status header, attention merge counters (zero between
// calls), then one region shared by the indexer's buffers and the attention
// partials (the two calls run one after the other).
constexpr int kPrefillMaxT = 1 << 18;

struct PrefillLayout {
    size_t status = 0;
    size_t counters = 0;
    size_t region = 0;
    size_t pm = 0, pl = 0, po = 0;
    size_t total = 0;
    lsa::PrefillPlan P{};
    lsa::AttnPlan A{};
};

PrefillLayout prefill_layout(const lsa_dims* d, int nq, int B, int num_sms) {
    PrefillLayout L;
    size_t off = kHeaderBytes;
    L.counters = off;
    off = align_up(off + (size_t)nq * d->hkv * 4);
    L.region = off;
    L.P = lsa::plan_prefill(d->hq, d->hkv, d->r, d->T, nq, B);
    const size_t index_end = L.region + L.P.bytes;
    const int G = d->hq / d->hkv;
    L.A = lsa::plan_attn(nq, d->hkv, G, B, d->d, num_sms);
    const size_t slots = (size_t)L.A.units * L.A.smax * G;
    L.pm = L.region;
    L.pl = L.pm + align_up(slots * 4);
    L.po = L.pl + align_up(slots * 4);
    const size_t attn_end = L.po + align_up(slots * (size_t)d->d * 4);
    L.total = align_up(index_end > attn_end ? index_end : attn_end);
    return L;
}

lsa_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
    if (!ws) return LSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return LSA_ERR_WORKSPACE;
    if (ws_bytes < need) return LSA_ERR_WORKSPACE;
    return LSA_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

// Scratch of lsa_indexed_attn_noalloc: one fixed buffer per device, part of
// this module's device image, so that the call never allocates. Byte layout
// of one call: merge counters [units] uint32 at offset 0 (zero between
// calls), then pm, pl [slots] fp32 and po [slots, d] fp32, each 256-aligned.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LSA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device. The first call per
// device looks it up and zero-fills the buffer on `stream`, waiting for it.
lsa_status noalloc_scratch(cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSA_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
            return LSA_ERR_CUDA;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LSA_ERR_CUDA;
        if (cudaMemsetAsync(p, 0, LSA_NOALLOC_SCRATCH_BYTES, stream) != cudaSuccess) return LSA_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return LSA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" {

int lsa_version(void) { return 100; }

const char* lsa_status_string(lsa_status s) {
    switch (s) {
        case LSA_OK: return "LSA_OK";
        case LSA_ERR_ARG: return "LSA_ERR_ARG: invalid argument (null pointer or bad size)";
        case LSA_ERR_ALIGN: return "LSA_ERR_ALIGN: pointer not 16-byte aligned";
        case LSA_ERR_SHAPE: return "LSA_ERR_SHAPE: inconsistent sizes";
        case LSA_ERR_WORKSPACE: return "LSA_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case LSA_ERR_CUDA: return "LSA_ERR_CUDA: a CUDA launch failed";
        case LSA_ERR_TIMEOUT: return "LSA_ERR_TIMEOUT: a device-side wait ran out";
        case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED: sizes outside the supported set";
        case LSA_ERR_SCRATCH:
            return "LSA_ERR_SCRATCH: sizes need more than the fixed no-alloc scratch (LSA_NOALLOC_SCRATCH_BYTES)";
        default: return "LSA_ERR_UNKNOWN";
    }
}

void lsa_debug_set_wait_limit(long long ns) { g_wait_limit.store(ns < 0 ? kDefaultWaitLimit : ns); }

size_t lsa_workspace_size(const lsa_dims* dims, int B, int blk, int nblk_keep) {
    if (check_dims(dims) != LSA_OK || check_B_attn(B) != LSA_OK) return 0;
    if (blk < 0 || nblk_keep < 0 || (blk > 0) != (nblk_keep > 0)) return 0;
    return decode_layout(dims, B, blk, nblk_keep, device_sms()).total;
}

lsa_status lsa_score(const lsa_dims* dims, const lsa_bf16* qt, const lsa_bf16* kt, float* scores, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if (!qt || !kt || !scores) return LSA_ERR_ARG;
    if (!aligned16(qt) || !aligned16(kt) || !aligned16(scores)) return LSA_ERR_ALIGN;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(lsa::launch_score(ctx, qt, kt, scores, dims->batch, dims->hq, dims->hkv, dims->r, dims->T, 1,
                                       nullptr));
}

lsa_status lsa_topk(const lsa_dims* dims, const float* scores, int B, int32_t* idx, void* ws, size_t ws_bytes,
                    void* stream) {
    (void)ws;
    (void)ws_bytes;
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!scores || !idx) return LSA_ERR_ARG;
    if (!aligned16(scores) || !aligned16(idx)) return LSA_ERR_ALIGN;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(
        lsa::launch_topk(ctx, scores, dims->batch * dims->hkv, dims->T, B, idx, nullptr, 0, 0));
}

lsa_status lsa_indexed_attn(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k, const lsa_bf16* v,
                            const int32_t* idx, int B, float scale, lsa_bf16* out, void* ws, size_t ws_bytes,
                            void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B_attn(B)) != LSA_OK) return s;
    if (!q || !k || !v || !idx || !out) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out)) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const DecodeLayout L = decode_layout(dims, B, 0, 0, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    return from_cuda(lsa::launch_attn(ctx, L.plan, q, k, v, idx, B, scale, out, at<float>(ws, L.pm),
                                      at<float>(ws, L.pl), at<float>(ws, L.po),
                                      at<unsigned>(ws, L.counters), dims->batch, dims->hq, dims->hkv,
                                      dims->d, dims->T, (long long)dims->T * dims->hkv,
                                      at<unsigned>(ws, L.status)));
}

lsa_status lsa_indexed_attn_noalloc(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k, const lsa_bf16* v,
                                    const int32_t* idx, int B, float scale, lsa_bf16* out, int32_t* dev_status,
                                    void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B_attn(B)) != LSA_OK) return s;
    if (!q || !k || !v || !idx || !out) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out)) return LSA_ERR_ALIGN;
    if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const int G = dims->hq / dims->hkv;
    const lsa::AttnPlan plan = lsa::plan_attn(dims->batch, dims->hkv, G, B, dims->d, ctx.num_sms);
    const size_t slots = (size_t)plan.units * plan.smax * G;
    const size_t pm = align_up((size_t)plan.units * 4);
    const size_t pl = pm + align_up(slots * 4);
    const size_t po = pl + align_up(slots * 4);
    const size_t need = po + align_up(slots * (size_t)dims->d * 4);
    if (need > LSA_NOALLOC_SCRATCH_BYTES) return LSA_ERR_SCRATCH;
    void* base = nullptr;
    if ((s = noalloc_scratch(ctx.stream, &base)) != LSA_OK) return s;
    return from_cuda(lsa::launch_attn(ctx, plan, q, k, v, idx, B, scale, out, at<float>(base, pm),
                                      at<float>(base, pl), at<float>(base, po), at<unsigned>(base, 0),
                                      dims->batch, dims->hq, dims->hkv, dims->d, dims->T,
                                      (long long)dims->T * dims->hkv, reinterpret_cast<unsigned*>(dev_status)));
}

lsa_status lsa_decode_step(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt, const lsa_bf16* k,
                           const lsa_bf16* v, const lsa_bf16* kt, const lsa_bf16* centroids, int blk, int nblk_keep,
                           int B, float scale, int32_t* idx_out, lsa_bf16* out, void* ws, size_t ws_bytes,
                           void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!q || !qt || !k || !v || !kt || !out) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(qt) || !aligned16(k) || !aligned16(v) || !aligned16(kt) || !aligned16(out))
        return LSA_ERR_ALIGN;
    if (idx_out && !aligned16(idx_out)) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const bool hier = centroids != nullptr;
    if (hier) {
        if (!aligned16(centroids)) return LSA_ERR_ALIGN;
        if (blk < 1 || blk > 4096 || nblk_keep < 1) return LSA_ERR_ARG;
        if ((long long)nblk_keep * blk > (1ll << 24)) return LSA_ERR_UNSUPPORTED;
        const int nblk = (dims->T + blk - 1) / blk;
        if (nblk_keep > nblk) nblk_keep = nblk;
    } else {
        blk = 0;
        nblk_keep = 0;
    }
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const DecodeLayout L = decode_layout(dims, B, blk, nblk_keep, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    unsigned* status = at<unsigned>(ws, L.status);
    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    const int rows = dims->batch * dims->hkv;
    cudaError_t e;
    if (!hier) {
        bool hist = false;
        uint32_t* gh = at<uint32_t>(ws, L.hist);
        e = lsa::launch_score(ctx, qt, kt, at<float>(ws, L.scores), dims->batch, dims->hq, dims->hkv, dims->r, dims->T,
                              0, status, gh, &hist);
        if (e == cudaSuccess)
            e = lsa::launch_topk(ctx, at<float>(ws, L.scores), rows, dims->T, B, idx, nullptr, 0, 0,
                                 hist ? gh : nullptr);
    } else {
        const int nblk = (dims->T + blk - 1) / blk;
        int32_t* blkidx = at<int32_t>(ws, L.blkidx);
        float* fine = at<float>(ws, L.fine);
        bool hist = false;
        uint32_t* gh = at<uint32_t>(ws, L.hist);
        e = lsa::launch_score(ctx, qt, centroids, at<float>(ws, L.scores), dims->batch, dims->hq, dims->hkv, dims->r,
                              nblk, 0, status, gh, &hist);
        if (e == cudaSuccess)
            e = lsa::launch_topk(ctx, at<float>(ws, L.scores), rows, nblk, nblk_keep, blkidx, nullptr, 0, 0,
                                 hist ? gh : nullptr);
        if (e == cudaSuccess)
            e = lsa::launch_fine_score(ctx, qt, kt, blkidx, nblk_keep, blk, fine, dims->batch, dims->hq, dims->hkv,
                                       dims->r, dims->T);
        if (e == cudaSuccess)
            e = lsa::launch_topk(ctx, fine, rows, nblk_keep * blk, B, idx, blkidx, blk, nblk_keep);
    }
    if (e == cudaSuccess)
        e = lsa::launch_attn(ctx, L.plan, q, k, v, idx, B, scale, out, at<float>(ws, L.pm), at<float>(ws, L.pl),
                             at<float>(ws, L.po), at<unsigned>(ws, L.counters), dims->batch, dims->hq,
                             dims->hkv, dims->d, dims->T,
                             (long long)dims->T * dims->hkv, status);
    return from_cuda(e);
}

lsa_status lsa_indexed_attn_paged(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* k_pool,
                                  const lsa_bf16* v_pool, int nslots, const int32_t* page_table, const int32_t* idx,
                                  int B, float scale, lsa_bf16* out, void* ws, size_t ws_bytes, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B_attn(B)) != LSA_OK) return s;
    if (!q || !k_pool || !v_pool || !page_table || !idx || !out || nslots < 1) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(page_table) || !aligned16(idx) ||
        !aligned16(out))
        return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const DecodeLayout L = decode_layout(dims, B, 0, 0, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    return from_cuda(lsa::launch_attn(ctx, L.plan, q, k_pool, v_pool, idx, B, scale, out, at<float>(ws, L.pm),
                                      at<float>(ws, L.pl), at<float>(ws, L.po), at<unsigned>(ws, L.counters),
                                      dims->batch, dims->hq, dims->hkv, dims->d, dims->T, 0,
                                      at<unsigned>(ws, L.status), page_table, nslots));
}

lsa_status lsa_decode_step_paged(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt, const lsa_bf16* k_pool,
                                 const lsa_bf16* v_pool, int nslots, const int32_t* page_table, const lsa_bf16* kt,
                                 int B, float scale, int32_t* idx_out, lsa_bf16* out, void* ws, size_t ws_bytes,
                                 void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!q || !qt || !k_pool || !v_pool || !page_table || !kt || !out || nslots < 1) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(qt) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(page_table) ||
        !aligned16(kt) || !aligned16(out))
        return LSA_ERR_ALIGN;
    if (idx_out && !aligned16(idx_out)) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const DecodeLayout L = decode_layout(dims, B, 0, 0, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    unsigned* status = at<unsigned>(ws, L.status);
    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    bool hist = false;
    uint32_t* gh = at<uint32_t>(ws, L.hist);
    cudaError_t e = lsa::launch_score(ctx, qt, kt, at<float>(ws, L.scores), dims->batch, dims->hq, dims->hkv, dims->r,
                                      dims->T, 0, status, gh, &hist);
    if (e == cudaSuccess)
        e = lsa::launch_topk(ctx, at<float>(ws, L.scores), dims->batch * dims->hkv, dims->T, B, idx, nullptr, 0, 0,
                             hist ? gh : nullptr);
    if (e == cudaSuccess)
        e = lsa::launch_attn(ctx, L.plan, q, k_pool, v_pool, idx, B, scale, out, at<float>(ws, L.pm),
                             at<float>(ws, L.pl), at<float>(ws, L.po), at<unsigned>(ws, L.counters), dims->batch,
                             dims->hq, dims->hkv, dims->d, dims->T, 0, status, page_table, nslots);
    return from_cuda(e);
}

static bool fp8_shape_ok(const lsa_dims* d) {
    return d->r == 64 && (d->hkv == 4 || d->hkv == 8 || d->hkv == 16 || d->hkv == 32);
}

lsa_status lsa_score_fp8(const lsa_dims* dims, const lsa_bf16* qt, const lsa_fp8_e4m3* kt, float* scores,
                         void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if (!fp8_shape_ok(dims)) return LSA_ERR_UNSUPPORTED;
    if (!qt || !kt || !scores) return LSA_ERR_ARG;
    if (!aligned16(qt) || !aligned16(kt) || !aligned16(scores)) return LSA_ERR_ALIGN;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(lsa::launch_score_fp8(ctx, qt, kt, scores, dims->batch, dims->hq, dims->hkv, dims->r, dims->T, 1,
                                           nullptr));
}

lsa_status lsa_decode_step_fp8(const lsa_dims* dims, const lsa_bf16* q, const lsa_bf16* qt, const lsa_bf16* k,
                               const lsa_bf16* v, const lsa_fp8_e4m3* kt, int B, float scale, int32_t* idx_out,
                               lsa_bf16* out, void* ws, size_t ws_bytes, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!fp8_shape_ok(dims)) return LSA_ERR_UNSUPPORTED;
    if (!q || !qt || !k || !v || !kt || !out) return LSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(qt) || !aligned16(k) || !aligned16(v) || !aligned16(kt) || !aligned16(out))
        return LSA_ERR_ALIGN;
    if (idx_out && !aligned16(idx_out)) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const DecodeLayout L = decode_layout(dims, B, 0, 0, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    unsigned* status = at<unsigned>(ws, L.status);
    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    bool hist = false;
    uint32_t* gh = at<uint32_t>(ws, L.hist);
    cudaError_t e = lsa::launch_score_fp8(ctx, qt, kt, at<float>(ws, L.scores), dims->batch, dims->hq, dims->hkv,
                                          dims->r, dims->T, 0, status, gh, &hist);
    if (e == cudaSuccess)
        e = lsa::launch_topk(ctx, at<float>(ws, L.scores), dims->batch * dims->hkv, dims->T, B, idx, nullptr, 0, 0,
                             hist ? gh : nullptr);
    if (e == cudaSuccess)
        e = lsa::launch_attn(ctx, L.plan, q, k, v, idx, B, scale, out, at<float>(ws, L.pm), at<float>(ws, L.pl),
                             at<float>(ws, L.po), at<unsigned>(ws, L.counters), dims->batch, dims->hq, dims->hkv,
                             dims->d, dims->T, (long long)dims->T * dims->hkv, status);
    return from_cuda(e);
}

lsa_status lsa_block_centroids(const lsa_dims* dims, const lsa_bf16* kt, int blk, lsa_bf16* centroids, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if (!kt || !centroids) return LSA_ERR_ARG;
    if (blk < 1 || blk > 4096) return LSA_ERR_ARG;
    if (!aligned16(kt) || !aligned16(centroids)) return LSA_ERR_ALIGN;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(lsa::launch_centroids(ctx, kt, blk, centroids, dims->batch, dims->hkv, dims->r, dims->T));
}

static lsa_status project_common(const lsa_proj_dims* pd, const lsa_bf16* x, const lsa_bf16* P, int t0, int n,
                                 void* y, bool fp8, int32_t* dev_status, void* stream) {
    if (!pd || !x || !P || !y) return LSA_ERR_ARG;
    if (pd->batch < 1 || pd->T < 1 || pd->H < 1 || pd->d < 1 || pd->r < 1 || pd->nbases < 1) return LSA_ERR_ARG;
    if (pd->H % pd->nbases != 0) return LSA_ERR_ARG;
    if (t0 < 0 || n < 0 || (long long)t0 + n > pd->T) return LSA_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(P) || !aligned16(y)) return LSA_ERR_ALIGN;
    if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return LSA_ERR_ALIGN;
    const int d = pd->d, r = pd->r;
    const bool d_ok = d % 16 == 0 && (d == 16 || d == 32 || (d >= 64 && d <= 256));
    const bool r_ok = r % 16 == 0 && r >= 16 && r <= 128;
    if (!d_ok || !r_ok || (long long)pd->batch * pd->T >= (1ll << 31) || lsa::project_stages(d, r, 2) < 2)
        return LSA_ERR_UNSUPPORTED;
    if (n == 0) return LSA_OK;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(lsa::launch_project(ctx, x, P, y, fp8, pd->batch, pd->T, pd->H, d, r, pd->nbases, t0, n,
                                         reinterpret_cast<unsigned*>(dev_status)));
}

lsa_status lsa_project(const lsa_proj_dims* dims, const lsa_bf16* x, const lsa_bf16* P, int t0, int n, lsa_bf16* y,
                       int32_t* dev_status, void* stream) {
    return project_common(dims, x, P, t0, n, y, false, dev_status, stream);
}

lsa_status lsa_project_fp8(const lsa_proj_dims* dims, const lsa_bf16* x, const lsa_bf16* P, int t0, int n,
                           lsa_fp8_e4m3* y, int32_t* dev_status, void* stream) {
    return project_common(dims, x, P, t0, n, y, true, dev_status, stream);
}

lsa_status lsa_update_centroids(const lsa_dims* dims, const lsa_bf16* kt, int blk, int t0, int n,
                                lsa_bf16* centroids, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if (!kt || !centroids) return LSA_ERR_ARG;
    if (blk < 1 || blk > 4096) return LSA_ERR_ARG;
    if (t0 < 0 || n < 0 || (long long)t0 + n > dims->T) return LSA_ERR_SHAPE;
    if (!aligned16(kt) || !aligned16(centroids)) return LSA_ERR_ALIGN;
    if (n == 0) return LSA_OK;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    return from_cuda(lsa::launch_centroid_update(ctx, kt, centroids, dims->batch, dims->T, dims->hkv, dims->r, blk,
                                                 t0, n));
}

size_t lsa_prefill_workspace_size(const lsa_dims* dims, int nq, int B) {
    if (check_dims(dims) != LSA_OK || check_B(B) != LSA_OK || nq < 1 || dims->batch != 1) return 0;
    return prefill_layout(dims, nq, B, device_sms()).total;
}

lsa_status lsa_prefill_index(const lsa_dims* dims, const lsa_bf16* qt, int nq, int q_start, const lsa_bf16* kt, int B,
                             int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!qt || !kt || !idx || nq < 1 || q_start < 0) return LSA_ERR_ARG;
    if (dims->batch != 1 || (long long)q_start + nq > dims->T) return LSA_ERR_SHAPE;
    if (dims->T > kPrefillMaxT) return LSA_ERR_UNSUPPORTED;
    if (!aligned16(qt) || !aligned16(kt) || !aligned16(idx)) return LSA_ERR_ALIGN;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const PrefillLayout L = prefill_layout(dims, nq, B, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    return from_cuda(lsa::launch_prefill_index(ctx, L.P, qt, kt, dims->hq, dims->hkv, dims->r, dims->T, nq, q_start, B,
                                               idx, at<uint8_t>(ws, L.region), at<unsigned>(ws, L.status)));
}

lsa_status lsa_prefill_attn(const lsa_dims* dims, const lsa_bf16* q, int nq, const lsa_bf16* k, const lsa_bf16* v,
                            const int32_t* idx, int B, float scale, lsa_bf16* out, void* ws, size_t ws_bytes,
                            void* stream) {
    lsa_status s = check_dims(dims);
    if (s != LSA_OK) return s;
    if ((s = check_B(B)) != LSA_OK) return s;
    if (!q || !k || !v || !idx || !out || nq < 1) return LSA_ERR_ARG;
    if (dims->batch != 1) return LSA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out)) return LSA_ERR_ALIGN;
    if (!std::isfinite(scale)) return LSA_ERR_ARG;
    const lsa::LaunchCtx ctx = make_ctx(stream);
    const PrefillLayout L = prefill_layout(dims, nq, B, ctx.num_sms);
    if ((s = check_ws(ws, ws_bytes, L.total)) != LSA_OK) return s;
    return from_cuda(lsa::launch_attn(ctx, L.A, q, k, v, idx, B, scale, out, at<float>(ws, L.pm), at<float>(ws, L.pl),
                                      at<float>(ws, L.po), at<unsigned>(ws, L.counters), nq, dims->hq, dims->hkv,
                                      dims->d, dims->T, 0, at<unsigned>(ws, L.status)));
}

lsa_status lsa_read_device_status(const void* ws, int32_t* host_flags, void* stream) {
    if (!ws || !host_flags) return LSA_ERR_ARG;
    return from_cuda(cudaMemcpyAsync(host_flags, ws, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

lsa_status lsa_clear_device_status(void* ws, void* stream) {
    if (!ws) return LSA_ERR_ARG;
    return from_cuda(cudaMemsetAsync(ws, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
