// stq_api.cu -- host side of the C ABI declared in include/stq.h:
// pool allocation and tables, argument checking, status and error strings,
// slot export/import, the device error word, host-side fault injection.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "stq_internal.h"

struct stq_pool {
    int kind = 0, R = 0, S = 0, H = 0;
    int scale_bytes = 4, raw_bits = 0;
    bool pivots = false;       // FP16 pivot units among quantized ones
    bool pivot_heads = false;  // GDN pivot heads (their own kernel)
    int n_pivot_heads = 0;
    bool fit = false;          // per-page column factors refitted at every quantisation
    bool per_row = false;      // KDA: every tile on the decode kernel's per-row path
    int device = 0;
    size_t slot_bytes = 0, packed_bytes = 0;
    uint8_t *d_pages = nullptr;
    void *d_tables = nullptr;
    uint32_t *d_err = nullptr;
    // debug checks (STQ_DEBUG_CHECKS=1 at creation): one bit per (request, slot)
    bool check_dups = false;
    uint32_t *d_seen = nullptr;
    // split decode: events behind the last readout and the last write-back
    cudaEvent_t ev_read = nullptr, ev_wb = nullptr;
    mutable bool wb_pending = false;
    // host-buffer decode: device staging, and an event behind its last use
    uint8_t *h_stage = nullptr;
    size_t h_stage_bytes = 0;
    cudaEvent_t h_done = nullptr;
    bool h_used = false;
    stq::Tables t{};
    std::vector<uint32_t> head_off, page_bytes;
};

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

stq_status fail(stq_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

stq_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(e == cudaErrorMemoryAllocation ? STQ_ERR_OOM : STQ_ERR_CUDA, "%s: %s", what,
                cudaGetErrorString(e));
}

bool fault(const char *which)
{
    const char *f = std::getenv("STQ_FAULT");
    return f != nullptr && std::strcmp(f, which) == 0;
}

// Layout of one head's page from its row bit widths and the bytes per row
// scale (4 fp32, 2 binary16, 0 for a raw page).
struct HeadLayout {
    uint32_t page_bytes;
    uint16_t row_off[stq::kD];
};

HeadLayout head_layout(const uint8_t *row_bits, int scale_bytes, bool fit)
{
    HeadLayout L{};
    uint32_t off = (uint32_t)scale_bytes * stq::kD + (fit ? (uint32_t)stq::kFitBytes : 0u);
    for (int i = 0; i < stq::kD; ++i) {
        L.row_off[i] = (uint16_t)off;
        off += 16u * row_bits[i];
    }
    L.page_bytes = (off + stq::kPageAlign - 1) / stq::kPageAlign * stq::kPageAlign;
    return L;
}

// Width of a raw pool (every unit 16, or every unit 32 bits), else 0.
int raw_width_of(const stq_pool_desc *d)
{
    const size_t nunits = d->kind == STQ_GDN ? (size_t)d->num_heads : (size_t)d->num_heads * stq::kD;
    const int b0 = d->unit_bits[0];
    if (b0 != 16 && b0 != 32) return 0;
    for (size_t u = 1; u < nunits; ++u)
        if (d->unit_bits[u] != b0) return 0;
    return b0;
}

// Bytes per row scale of a (validated) description: 0 for a raw pool.
int scale_bytes_of(const stq_pool_desc *d)
{
    if (raw_width_of(d)) return 0;
    return (d->flags & STQ_SCALE_F16) ? 2 : 4;
}

// Validates a description; fills the per-row bit table [H][128].
stq_status check_desc(const stq_pool_desc *d, std::vector<uint8_t> *row_bits)
{
    if (d == nullptr) return fail(STQ_ERR_ARG, "desc is NULL");
    if (d->kind != STQ_GDN && d->kind != STQ_KDA) return fail(STQ_ERR_ARG, "kind %d", d->kind);
    if (d->num_requests < 1 || d->num_slots < 1 || d->num_heads < 1)
        return fail(STQ_ERR_ARG, "sizes R=%d S=%d H=%d must be >= 1", d->num_requests,
                    d->num_slots, d->num_heads);
    if (d->d_k != stq::kD || d->d_v != stq::kD)
        return fail(STQ_ERR_UNSUPPORTED, "d_k=%d d_v=%d: only 128 x 128 states", d->d_k, d->d_v);
    if (d->unit_bits == nullptr) return fail(STQ_ERR_ARG, "unit_bits is NULL");
    const int H = d->num_heads;
    const size_t nunits = d->kind == STQ_GDN ? (size_t)H : (size_t)H * stq::kD;
    if (d->flags & ~(STQ_SCALE_F16 | STQ_FIT_COLUMNS)) return fail(STQ_ERR_ARG, "flags 0x%x", d->flags);
    for (size_t u = 0; u < nunits; ++u) {
        int b = d->unit_bits[u];
        if (b != 4 && b != 6 && b != 8 && b != 16 && b != 32)
            return fail(STQ_ERR_ARG, "unit_bits[%zu] = %d (must be 4, 6, 8, 16 or 32)", u, b);
    }
    const int raw = raw_width_of(d);
    if (!raw)
        for (size_t u = 0; u < nunits; ++u)
            if (d->unit_bits[u] == 32)
                return fail(STQ_ERR_UNSUPPORTED, "unit_bits[%zu] = 32: fp32 units must make up the whole pool", u);
    if (raw && d->flags != 0) return fail(STQ_ERR_ARG, "a raw pool has no scales (flags must be 0)");
    if ((d->flags & STQ_FIT_COLUMNS) && d->row_weight)
        for (size_t e = 0; e < (size_t)H * stq::kD; ++e)
            if (!(std::isfinite(d->row_weight[e]) && d->row_weight[e] > 0.0f))
                return fail(STQ_ERR_ARG, "row_weight[%zu] = %g (must be finite and > 0)", e, (double)d->row_weight[e]);
    for (int which = 0; which < 2; ++which) {
        const float *f = which ? d->col_factor : d->row_factor;
        if (f == nullptr) continue;
        for (size_t e = 0; e < (size_t)H * stq::kD; ++e)
            if (!(std::isfinite(f[e]) && f[e] > 0.0f))
                return fail(STQ_ERR_ARG, "%s_factor[%zu] = %g (must be finite and > 0)",
                            which ? "col" : "row", e, (double)f[e]);
    }
    if (row_bits) {
        row_bits->resize((size_t)H * stq::kD);
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < stq::kD; ++i)
                (*row_bits)[(size_t)h * stq::kD + i] =
                    d->kind == STQ_GDN ? d->unit_bits[h] : d->unit_bits[(size_t)h * stq::kD + i];
    }
    return STQ_OK;
}

stq_status sizes_of(const stq_pool_desc *d, const std::vector<uint8_t> &row_bits,
                    std::vector<uint32_t> *head_off, std::vector<uint32_t> *page_bytes,
                    size_t *slot_bytes, size_t *packed)
{
    size_t off = 0;
    const int sb = scale_bytes_of(d);
    for (int h = 0; h < d->num_heads; ++h) {
        HeadLayout L = head_layout(&row_bits[(size_t)h * stq::kD], sb, (d->flags & STQ_FIT_COLUMNS) != 0);
        if (d->kind == STQ_KDA && sb != 0 && L.page_bytes > (uint32_t)stq::kMaxStagedPage)
            return fail(STQ_ERR_UNSUPPORTED, "KDA head %d: %u-byte page (FP16 pivot rows average above 8 bits "
                        "per row); at most %d bytes", h, L.page_bytes, stq::kMaxStagedPage);
        if (head_off) head_off->push_back((uint32_t)off);
        if (page_bytes) page_bytes->push_back(L.page_bytes);
        off += L.page_bytes;
        if (off > 0xFFFFFFFFull) return fail(STQ_ERR_UNSUPPORTED, "slot larger than 4 GiB");
    }
    const double total = (double)off * d->num_requests * d->num_slots;
    if (total > 9.0e18) return fail(STQ_ERR_ARG, "pool size overflows");
    *slot_bytes = off;
    *packed = off * (size_t)d->num_requests * (size_t)d->num_slots;
    return STQ_OK;
}

stq::PoolView view(stq_pool *p)
{
    stq::PoolView v;
    v.pages = p->d_pages;
    v.slot_bytes = p->slot_bytes;
    v.R = p->R;
    v.S = p->S;
    v.H = p->H;
    v.kind = p->kind;
    v.scale_bytes = p->scale_bytes;
    v.raw_bits = p->raw_bits;
    v.pivots = p->pivots ? 1 : 0;
    v.fit = p->fit ? 1 : 0;
    v.per_row = p->per_row ? 1 : 0;
    v.n_pivot_heads = p->n_pivot_heads;
    v.t = p->t;
    v.err = p->d_err;
    // STQ_FAULT=timeout: a wait that nothing completes, given a short limit
    const bool stall = fault("timeout");
    v.wait_ns = stall ? 2000000ull : 1000000000ull;
    v.stall_tx = stall ? 16u : 0u;
    return v;
}

// An NVTX range over a launching call (a no-op unless a profiler is attached),
// so that profiles attribute device work to the entry point that queued it.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Makes the pool's device current for the duration of a call.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            ok = false;
            return;
        }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

stq_status check_launch_args(const stq_pool *p, const int32_t *req, const int32_t *slot, int32_t n)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    if (n < 0) return fail(STQ_ERR_ARG, "n = %d", n);
    if (n > 0 && (req == nullptr || slot == nullptr))
        return fail(STQ_ERR_ARG, "req_idx / slot_idx is NULL");
    if ((long long)n * p->H > 0x7FFFFFFFll) return fail(STQ_ERR_ARG, "n * H too large");
    return STQ_OK;
}

// A pending split write-back is ordered before the next access: asynchronous
// calls make their stream wait for it, synchronous ones wait on the host.
cudaError_t join_async(const stq_pool *p, cudaStream_t stream)
{
    if (!p->wb_pending) return cudaSuccess;
    cudaError_t e = cudaStreamWaitEvent(stream, p->ev_wb, 0);
    if (e == cudaSuccess) p->wb_pending = false;
    return e;
}

// With debug checks on: flag (request, slot) pairs named twice in one call.
cudaError_t debug_checks(const stq_pool *p, const int32_t *req, const int32_t *slot, int32_t n, cudaStream_t s)
{
    if (!p->check_dups || n == 0) return cudaSuccess;
    return stq::launch_duplicate_check(req, slot, n, p->R, p->S, p->d_seen, p->d_err, s);
}

cudaError_t join_host(const stq_pool *p)
{
    if (!p->wb_pending) return cudaSuccess;
    cudaError_t e = cudaEventSynchronize(p->ev_wb);
    if (e == cudaSuccess) p->wb_pending = false;
    return e;
}

stq_status check_decode_args(const stq_pool *p, const int32_t *req, const int32_t *slot, int32_t n,
                             const float *q, const float *k, const float *v, const float *beta,
                             const float *gate, const float *y)
{
    stq_status st = check_launch_args(p, req, slot, n);
    if (st != STQ_OK) return st;
    if (n > 0 && (!q || !k || !v || !beta || !gate || !y))
        return fail(STQ_ERR_ARG, "a q/k/v/beta/gate/y pointer is NULL");
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) |
                          (p->kind == STQ_KDA ? reinterpret_cast<uintptr_t>(gate) : 0);
    if (mis % 16 != 0) return fail(STQ_ERR_ARG, "q, k, v (and the KDA gate) must be 16-byte aligned");
    return STQ_OK;
}

stq_status check_split_args(const stq_pool *p, int32_t n, const float *u_tilde)
{
    if (p->raw_bits) return fail(STQ_ERR_UNSUPPORTED, "split decode needs a quantized pool");
    if (n > 0 && u_tilde == nullptr) return fail(STQ_ERR_ARG, "u_tilde is NULL");
    if (reinterpret_cast<uintptr_t>(u_tilde) % 16 != 0) return fail(STQ_ERR_ARG, "u_tilde not 16-byte aligned");
    return STQ_OK;
}

}  // namespace

namespace stq {
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

stq_status fail_status(stq_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}
}  // namespace stq

using stq::kD;

extern "C" {

const char *stq_status_str(stq_status s)
{
    switch (s) {
    case STQ_OK: return "STQ_OK";
    case STQ_ERR_ARG: return "STQ_ERR_ARG";
    case STQ_ERR_OOM: return "STQ_ERR_OOM";
    case STQ_ERR_CUDA: return "STQ_ERR_CUDA";
    case STQ_ERR_INDEX: return "STQ_ERR_INDEX";
    case STQ_ERR_NONFINITE: return "STQ_ERR_NONFINITE";
    case STQ_ERR_UNSUPPORTED: return "STQ_ERR_UNSUPPORTED";
    case STQ_ERR_TIMEOUT: return "STQ_ERR_TIMEOUT";
    }
    return "STQ_ERR_UNKNOWN";
}

const char *stq_last_error(void) { return g_last_error.c_str(); }

uint64_t stq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

stq_status stq_desc_bytes(const stq_pool_desc *desc, size_t *packed_bytes, size_t *per_slot_bytes)
{
    std::vector<uint8_t> rb;
    stq_status st = check_desc(desc, &rb);
    if (st != STQ_OK) return st;
    size_t slot = 0, packed = 0;
    st = sizes_of(desc, rb, nullptr, nullptr, &slot, &packed);
    if (st != STQ_OK) return st;
    if (packed_bytes) *packed_bytes = packed;
    if (per_slot_bytes) *per_slot_bytes = slot;
    return STQ_OK;
}

stq_status stq_pool_create(const stq_pool_desc *desc, stq_pool **out)
{
    if (out == nullptr) return fail(STQ_ERR_ARG, "out is NULL");
    *out = nullptr;
    std::vector<uint8_t> rb;
    stq_status st = check_desc(desc, &rb);
    if (st != STQ_OK) return st;
    if (fault("alloc")) return fail(STQ_ERR_OOM, "injected allocation failure (STQ_FAULT=alloc)");

    stq_pool *p = new stq_pool();
    p->kind = desc->kind;
    p->R = desc->num_requests;
    p->S = desc->num_slots;
    p->H = desc->num_heads;
    p->scale_bytes = scale_bytes_of(desc);
    p->raw_bits = raw_width_of(desc);
    for (size_t u = 0; !p->raw_bits && u < rb.size(); ++u) p->pivots |= rb[u] == 16;
    p->pivot_heads = p->pivots && p->kind == STQ_GDN;
    p->fit = (desc->flags & STQ_FIT_COLUMNS) != 0;
    st = sizes_of(desc, rb, &p->head_off, &p->page_bytes, &p->slot_bytes, &p->packed_bytes);
    if (st != STQ_OK) {
        delete p;
        return st;
    }
    const int H = p->H;
    // host image of the tables
    const size_t n_hoff = (size_t)H * 4, n_pb = (size_t)H * 4, n_ro = (size_t)H * kD * 2,
                 n_rb = (size_t)H * kD, n_f = (size_t)H * kD * 4;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t n_blk = (size_t)H * stq::kHeadBlock, n_ph = (size_t)H * 4;
    const size_t o_hoff = 0, o_pb = o_hoff + al(n_hoff), o_ro = o_pb + al(n_pb),
                 o_rb = o_ro + al(n_ro), o_r = o_rb + al(n_rb), o_c = o_r + al(n_f),
                 o_w = o_c + al(n_f), o_blk = o_w + al(n_f), o_ph = o_blk + al(n_blk),
                 total = o_ph + al(n_ph);
    std::vector<uint8_t> img(total, 0);
    std::memcpy(&img[o_hoff], p->head_off.data(), n_hoff);
    std::memcpy(&img[o_pb], p->page_bytes.data(), n_pb);
    for (int h = 0; h < H; ++h) {
        HeadLayout L = head_layout(&rb[(size_t)h * kD], p->scale_bytes, p->fit);
        std::memcpy(&img[o_ro + (size_t)h * kD * 2], L.row_off, kD * 2);
    }
    std::memcpy(&img[o_rb], rb.data(), n_rb);
    if (p->pivot_heads) {
        // the GDN pivot heads (every row at 16 bits), so that their kernel launches only their tiles
        int32_t *ph = reinterpret_cast<int32_t *>(&img[o_ph]);
        for (int h = 0; h < H; ++h)
            if (rb[(size_t)h * kD] == 16) ph[p->n_pivot_heads++] = h;
    }
    float *fr = reinterpret_cast<float *>(&img[o_r]);
    float *fc = reinterpret_cast<float *>(&img[o_c]);
    float *fw = reinterpret_cast<float *>(&img[o_w]);  // w_i, the column fit's row weights (1 without)
    for (size_t e = 0; e < (size_t)H * kD; ++e) {
        fr[e] = desc->row_factor ? desc->row_factor[e] : 1.0f;
        fc[e] = desc->col_factor ? desc->col_factor[e] : 1.0f;
        fw[e] = (desc->flags & STQ_FIT_COLUMNS) && desc->row_weight ? desc->row_weight[e] : 1.0f;
    }
    for (int h = 0; h < H; ++h) {
        uint8_t *blk = &img[o_blk + (size_t)h * stq::kHeadBlock];
        std::memcpy(blk, fr + (size_t)h * kD, kD * 4);
        std::memcpy(blk + 512, fc + (size_t)h * kD, kD * 4);
        float inv_rq[kD];  // 1 / (r_i q_b(i)), rounded once from double; 1 / r_i for a pivot row (unused by raw pages)
        for (int i = 0; i < kD; ++i) {
            const int b = rb[(size_t)h * kD + i];
            const double r = (double)fr[(size_t)h * kD + i];
            inv_rq[i] = b <= 8 ? (float)(1.0 / (r * (double)((1 << (b - 1)) - 1))) : b == 16 ? (float)(1.0 / r) : 0.0f;
        }
        std::memcpy(blk + 1024, inv_rq, kD * 4);
        std::memcpy(blk + 1536, &img[o_ro + (size_t)h * kD * 2], kD * 2);
        std::memcpy(blk + 1792, &rb[(size_t)h * kD], kD);
        // the decode kernel's row order (position -> row): KDA rows sorted by width, so
        // that the two half-warps taking positions 16 w + 2 t and 16 w + 2 t + 1 at step t
        // of their rows mostly share a width; GDN rows in order
        uint8_t *perm = blk + 1920;
        int order[kD];
        for (int i = 0; i < kD; ++i) order[i] = i;
        const uint8_t *hb = &rb[(size_t)h * kD];
        if (p->kind == STQ_KDA) {
            std::stable_sort(order, order + kD, [hb](int a, int b) { return hb[a] < hb[b]; });
            for (int w = 0; w < 8; ++w)
                for (int g = 0; g < 2; ++g)
                    for (int t = 0; t < 8; ++t) perm[(2 * w + g) * 8 + t] = (uint8_t)order[16 * w + 2 * t + g];
            // a pass warp takes positions [16 w, 16 w + 16): the width-specialised passes need
            // one width of 4, 6 or 8 bits there; otherwise the whole pool takes the per-row path
            // (a launch mixing both kinds of pass measured slower than the per-row path alone)
            for (int w = 0; w < 8; ++w) {
                const int lo = hb[order[16 * w]], hi = hb[order[16 * w + 15]];
                if (lo != hi || lo > 8) p->per_row = true;
            }
        } else {
            for (int i = 0; i < kD; ++i) perm[i] = (uint8_t)i;
        }
    }

    cudaError_t e = cudaGetDevice(&p->device);
    if (e != cudaSuccess) {
        delete p;
        return cuda_fail(e, "cudaGetDevice");
    }
    e = cudaMalloc(&p->d_pages, p->packed_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_tables, total);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_err, 256);
    if (e == cudaSuccess) e = cudaMemset(p->d_pages, 0, p->packed_bytes);
    if (e == cudaSuccess) e = cudaMemset(p->d_err, 0, 256);
    if (e == cudaSuccess) e = cudaMemcpy(p->d_tables, img.data(), total, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && p->fit) {
        // a zero state still carries column factors: every page starts with the pool's
        // col_factor (the factors the first step takes its codes with, and refits)
        std::vector<uint8_t> slot(p->slot_bytes, 0);
        const float *fcs = reinterpret_cast<const float *>(&img[o_c]);
        for (int h = 0; h < H; ++h)
            std::memcpy(&slot[p->head_off[h] + (size_t)p->scale_bytes * kD], fcs + (size_t)h * kD, kD * 4);
        const size_t units = (size_t)p->R * p->S;
        e = cudaMemcpy(p->d_pages, slot.data(), p->slot_bytes, cudaMemcpyHostToDevice);
        for (size_t done = 1; e == cudaSuccess && done < units; done *= 2) {
            const size_t n = std::min(done, units - done);
            e = cudaMemcpy(p->d_pages + done * p->slot_bytes, p->d_pages, n * p->slot_bytes, cudaMemcpyDeviceToDevice);
        }
    }
    const char *dbg = std::getenv("STQ_DEBUG_CHECKS");
    p->check_dups = dbg != nullptr && std::strcmp(dbg, "1") == 0;
    if (e == cudaSuccess && p->check_dups)
        e = cudaMalloc(&p->d_seen, ((size_t)p->R * p->S + 31) / 32 * sizeof(uint32_t));
    if (e != cudaSuccess) {
        stq_status r = cuda_fail(e, "pool allocation");
        cudaFree(p->d_pages);
        cudaFree(p->d_tables);
        cudaFree(p->d_err);
        cudaFree(p->d_seen);
        cudaGetLastError();
        delete p;
        return r;
    }
    uint8_t *base = static_cast<uint8_t *>(p->d_tables);
    p->t.head_off = reinterpret_cast<const uint32_t *>(base + o_hoff);
    p->t.page_bytes = reinterpret_cast<const uint32_t *>(base + o_pb);
    p->t.row_off = reinterpret_cast<const uint16_t *>(base + o_ro);
    p->t.row_bits = base + o_rb;
    p->t.r = reinterpret_cast<const float *>(base + o_r);
    p->t.c = reinterpret_cast<const float *>(base + o_c);
    p->t.w = reinterpret_cast<const float *>(base + o_w);
    p->t.block = base + o_blk;
    p->t.pivot_head = reinterpret_cast<const int32_t *>(base + o_ph);
    *out = p;
    return STQ_OK;
}

stq_status stq_pool_destroy(stq_pool *p)
{
    if (p == nullptr) return STQ_OK;
    DeviceGuard g(p->device);
    if (p->wb_pending) cudaEventSynchronize(p->ev_wb);
    if (p->ev_read) cudaEventDestroy(p->ev_read);
    if (p->ev_wb) cudaEventDestroy(p->ev_wb);
    if (p->h_used) cudaEventSynchronize(p->h_done);
    if (p->h_done) cudaEventDestroy(p->h_done);
    cudaFree(p->h_stage);
    cudaFree(p->d_seen);
    cudaFree(p->d_pages);
    cudaFree(p->d_tables);
    cudaFree(p->d_err);
    delete p;
    return STQ_OK;
}

stq_status stq_pool_bytes(const stq_pool *p, size_t *packed_bytes, size_t *per_slot_bytes)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    if (packed_bytes) *packed_bytes = p->packed_bytes;
    if (per_slot_bytes) *per_slot_bytes = p->slot_bytes;
    return STQ_OK;
}

stq_status stq_page_layout(const stq_pool *p, int32_t head, size_t *offset_in_slot,
                           size_t *page_bytes)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    if (head < 0 || head >= p->H) return fail(STQ_ERR_ARG, "head %d out of [0, %d)", head, p->H);
    if (offset_in_slot) *offset_in_slot = p->head_off[head];
    if (page_bytes) *page_bytes = p->page_bytes[head];
    return STQ_OK;
}

stq_status stq_quantize_state(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                              int32_t n, const float *state, void *stream)
{
    stq_status st = check_launch_args(p, req_idx, slot_idx, n);
    if (st != STQ_OK) return st;
    if (n > 0 && state == nullptr) return fail(STQ_ERR_ARG, "state is NULL");
    if (reinterpret_cast<uintptr_t>(state) % 16 != 0) return fail(STQ_ERR_ARG, "state not 16-byte aligned");
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_quantize_state");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = debug_checks(p, req_idx, slot_idx, n, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "debug checks");
    e = stq::launch_quantize(view(p), req_idx, slot_idx, n, state, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "quantize launch");
}

stq_status stq_dequantize_state(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, float *state_out, void *stream)
{
    stq_status st = check_launch_args(p, req_idx, slot_idx, n);
    if (st != STQ_OK) return st;
    if (n > 0 && state_out == nullptr) return fail(STQ_ERR_ARG, "state_out is NULL");
    if (reinterpret_cast<uintptr_t>(state_out) % 16 != 0)
        return fail(STQ_ERR_ARG, "state_out not 16-byte aligned");
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_dequantize_state");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = stq::launch_dequantize(view(p), req_idx, slot_idx, n, state_out, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "dequantize launch");
}

stq_status stq_decode_step(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                           int32_t n, const float *q, const float *k, const float *v,
                           const float *beta, const float *gate, float *y, void *stream)
{
    stq_status st = check_decode_args(p, req_idx, slot_idx, n, q, k, v, beta, gate, y);
    if (st != STQ_OK) return st;
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_step");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = debug_checks(p, req_idx, slot_idx, n, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "debug checks");
    stq::DecodeIO io{req_idx, slot_idx, n, q, k, v, beta, gate, y, nullptr};
    e = p->raw_bits ? stq::launch_decode_raw(view(p), io, (cudaStream_t)stream)
                    : stq::launch_decode(view(p), io, (cudaStream_t)stream);
    if (e == cudaSuccess && p->pivot_heads) e = stq::launch_decode_pivot_heads(view(p), io, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "decode launch");
}

stq_status stq_decode_readout(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                              int32_t n, const float *q, const float *k, const float *v,
                              const float *beta, const float *gate, float *y, float *u_tilde,
                              void *stream)
{
    stq_status st = check_decode_args(p, req_idx, slot_idx, n, q, k, v, beta, gate, y);
    if (st != STQ_OK) return st;
    st = check_split_args(p, n, u_tilde);
    if (st != STQ_OK) return st;
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_readout");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    stq::DecodeIO io{req_idx, slot_idx, n, q, k, v, beta, gate, y, u_tilde};
    e = stq::launch_decode_readout(view(p), io, (cudaStream_t)stream);
    if (e == cudaSuccess && p->pivot_heads) e = stq::launch_decode_pivot_heads(view(p), io, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "readout launch");
}

stq_status stq_decode_writeback(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, const float *k, const float *gate,
                                const float *u_tilde, void *stream)
{
    stq_status st = check_launch_args(p, req_idx, slot_idx, n);
    if (st != STQ_OK) return st;
    if (n > 0 && (!k || !gate)) return fail(STQ_ERR_ARG, "k or gate is NULL");
    const uintptr_t mis = reinterpret_cast<uintptr_t>(k) |
                          (p->kind == STQ_KDA ? reinterpret_cast<uintptr_t>(gate) : 0);
    if (mis % 16 != 0) return fail(STQ_ERR_ARG, "k (and the KDA gate) must be 16-byte aligned");
    st = check_split_args(p, n, u_tilde);
    if (st != STQ_OK) return st;
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_writeback");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = debug_checks(p, req_idx, slot_idx, n, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "debug checks");
    // the write-back reads u~ through the v slot; q and beta are not read
    stq::DecodeIO io{req_idx, slot_idx, n, nullptr, k, u_tilde, nullptr, gate, nullptr, nullptr};
    e = stq::launch_decode_writeback(view(p), io, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "write-back launch");
}

stq_status stq_decode_step_split(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                                 int32_t n, const float *q, const float *k, const float *v,
                                 const float *beta, const float *gate, float *y, float *u_tilde,
                                 void *stream, void *side_stream)
{
    stq_status st = check_decode_args(p, req_idx, slot_idx, n, q, k, v, beta, gate, y);
    if (st != STQ_OK) return st;
    st = check_split_args(p, n, u_tilde);
    if (st != STQ_OK) return st;
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_step_split");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    cudaError_t e = cudaSuccess;
    if (p->ev_read == nullptr) e = cudaEventCreateWithFlags(&p->ev_read, cudaEventDisableTiming);
    if (e == cudaSuccess && p->ev_wb == nullptr) e = cudaEventCreateWithFlags(&p->ev_wb, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "event create");
    const cudaStream_t s0 = (cudaStream_t)stream, s1 = (cudaStream_t)side_stream;
    e = join_async(p, s0);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = debug_checks(p, req_idx, slot_idx, n, s0);
    if (e != cudaSuccess) return cuda_fail(e, "debug checks");
    stq::DecodeIO io{req_idx, slot_idx, n, q, k, v, beta, gate, y, u_tilde};
    e = stq::launch_decode_readout(view(p), io, s0);
    if (e == cudaSuccess && p->pivot_heads) e = stq::launch_decode_pivot_heads(view(p), io, s0);
    if (e != cudaSuccess) return cuda_fail(e, "readout launch");
    e = cudaEventRecord(p->ev_read, s0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s1, p->ev_read, 0);
    if (e != cudaSuccess) return cuda_fail(e, "readout event");
    stq::DecodeIO wb{req_idx, slot_idx, n, nullptr, k, u_tilde, nullptr, gate, nullptr, nullptr};
    e = stq::launch_decode_writeback(view(p), wb, s1);
    if (e != cudaSuccess) return cuda_fail(e, "write-back launch");
    e = cudaEventRecord(p->ev_wb, s1);
    if (e != cudaSuccess) return cuda_fail(e, "write-back event");
    p->wb_pending = true;
    return STQ_OK;
}

// ---------------------------------------------------------------- decode with built-in scratch
//
// The split step needs a per-tile u~ buffer between its two kernels.  Callers
// that cannot allocate device memory while they run (an engine that has
// reserved all of its device memory up front, or one whose latency budget
// cannot absorb an allocation, which may fail under memory pressure or wait
// for the whole device) can use stq_decode_step_static instead: it runs both
// kernels on one stream and keeps u~ in the fixed array below.  The array is
// part of the library's device image, so every GPU that loads the library
// holds its 4 MiB until the process exits.

}  // extern "C"

static __device__ __align__(256) float g_static_u_tilde[stq::kStaticScratchFloats];

namespace {

constexpr int kMaxScratchDevices = 64;
float *g_static_u_tilde_ptr[kMaxScratchDevices] = {};
std::mutex g_static_mu;

// Device address of the array on the current device.  In host code the
// array's name only stands for the symbol.  Outside stream capture the
// address is looked up on every call (so a context re-created after a device
// reset gets its own image's address) and cached per device; a call made
// while `stream` is being captured uses the cached address, which an earlier
// uncaptured call on this device must have set.
cudaError_t static_u_tilde(int dev, cudaStream_t stream, float **out)
{
    if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (cs == cudaStreamCaptureStatusNone || g_static_u_tilde_ptr[dev] == nullptr) {
        if (cs != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_u_tilde);
        if (e != cudaSuccess) return e;
        g_static_u_tilde_ptr[dev] = static_cast<float *>(ptr);
    }
    *out = g_static_u_tilde_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

stq_status stq_decode_step_static(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                                  int32_t n, const float *q, const float *k, const float *v,
                                  const float *beta, const float *gate, float *y, void *stream)
{
    stq_status st = check_decode_args(p, req_idx, slot_idx, n, q, k, v, beta, gate, y);
    if (st != STQ_OK) return st;
    if (p->raw_bits) return fail(STQ_ERR_UNSUPPORTED, "the built-in scratch decode needs a quantized pool");
    const long long need = (long long)n * p->H * kD;
    if (need > (long long)stq::kStaticScratchFloats)
        return fail(STQ_ERR_ARG, "n * H = %lld tiles exceeds the built-in scratch of %lld tiles",
                    (long long)n * p->H, (long long)(stq::kStaticScratchFloats / kD));
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_step_static");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    const cudaStream_t s0 = (cudaStream_t)stream;
    float *u = nullptr;
    cudaError_t e = static_u_tilde(p->device, s0, &u);
    if (e != cudaSuccess) return cuda_fail(e, "address of the built-in scratch");
    e = join_async(p, s0);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    e = debug_checks(p, req_idx, slot_idx, n, s0);
    if (e != cudaSuccess) return cuda_fail(e, "debug checks");
    // the readout fills u~ for every tile of the call before the write-back reads it
    stq::DecodeIO io{req_idx, slot_idx, n, q, k, v, beta, gate, y, u};
    e = stq::launch_decode_readout(view(p), io, s0);
    if (e == cudaSuccess && p->pivot_heads) e = stq::launch_decode_pivot_heads(view(p), io, s0);
    if (e != cudaSuccess) return cuda_fail(e, "readout launch");
    stq::DecodeIO wb{req_idx, slot_idx, n, nullptr, k, u, nullptr, gate, nullptr, nullptr};
    e = stq::launch_decode_writeback(view(p), wb, s0);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "write-back launch");
}

// ---------------------------------------------------------------- decode from host buffers
//
// Inputs in, one decode, y out, all on the caller's stream.  A page-locked y
// is written by the decode kernels themselves across the bus (each warp stores
// whole 128-byte lines), so it needs no copy back; a pageable y is staged and
// copied.  Cutting the entries into chunks pipelined over separate copy streams
// measured slower at 2048 tiles (each cross-stream wait costs more than the
// overlap it buys) and no faster at 8192, so the step stays on one stream.

}  // extern "C"

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of the staged arrays for n entries (each 256-byte aligned);
// the inputs end at `inputs`, y follows.
struct HostLayout {
    size_t req, slot, q, k, v, beta, gate, inputs, y, total;
};

HostLayout host_layout(const stq_pool *p, int32_t n)
{
    const size_t vec = (size_t)n * p->H * kD * sizeof(float), per = (size_t)n * p->H * sizeof(float);
    HostLayout L{};
    size_t o = 0;
    L.req = o;  o += align256((size_t)n * sizeof(int32_t));
    L.slot = o; o += align256((size_t)n * sizeof(int32_t));
    L.q = o;    o += align256(vec);
    L.k = o;    o += align256(vec);
    L.v = o;    o += align256(vec);
    L.beta = o; o += align256(per);
    L.gate = o; o += p->kind == STQ_KDA ? vec : per;
    L.inputs = o;
    o = align256(o);
    L.y = o;    o += align256(vec);
    L.total = o;
    return L;
}

// The staging buffer, at least `bytes` long, free for this call's stream to use.
cudaError_t host_staging(stq_pool *p, size_t bytes, cudaStream_t stream)
{
    cudaError_t e = cudaSuccess;
    if (p->h_done == nullptr) e = cudaEventCreateWithFlags(&p->h_done, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    if (bytes > p->h_stage_bytes) {
        // grow: the previous call's copies and launch must be done with the old buffer
        if (p->h_used) e = cudaEventSynchronize(p->h_done);
        if (e != cudaSuccess) return e;
        cudaFree(p->h_stage);
        p->h_stage = nullptr;
        p->h_stage_bytes = 0;
        p->h_used = false;
        const size_t grown = (bytes + (1u << 20) - 1) & ~static_cast<size_t>((1u << 20) - 1);
        e = cudaMalloc(&p->h_stage, grown);
        if (e == cudaSuccess) p->h_stage_bytes = grown;
        return e;
    }
    // the previous call may have run on another stream: wait for it unless it is done
    if (p->h_used && cudaEventQuery(p->h_done) != cudaSuccess) e = cudaStreamWaitEvent(stream, p->h_done, 0);
    return e;
}

// The step on inputs already copied into the staging buffer (queued on s0),
// with y written straight to a page-locked y or else copied back to the host;
// records the pool's staging event.
stq_status host_decode_and_copy_out(stq_pool *p, int32_t n, const HostLayout &L, float *y, cudaStream_t s0)
{
    uint8_t *d = p->h_stage;
    const size_t vec = (size_t)n * p->H * kD * sizeof(float);
    // page-locked y (device-addressable): the kernels write it directly, no copy back
    float *yk = reinterpret_cast<float *>(d + L.y);
    bool direct = false;
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, y) == cudaSuccess) {
        if (pa.type == cudaMemoryTypeHost && pa.devicePointer != nullptr) {
            yk = static_cast<float *>(pa.devicePointer);
            direct = true;
        }
    } else {
        cudaGetLastError();
    }
    const stq::DecodeIO io{reinterpret_cast<const int32_t *>(d + L.req), reinterpret_cast<const int32_t *>(d + L.slot),
                           n, reinterpret_cast<const float *>(d + L.q), reinterpret_cast<const float *>(d + L.k),
                           reinterpret_cast<const float *>(d + L.v), reinterpret_cast<const float *>(d + L.beta),
                           reinterpret_cast<const float *>(d + L.gate), yk, nullptr};
    cudaError_t e = debug_checks(p, io.req_idx, io.slot_idx, n, s0);
    if (e == cudaSuccess) e = p->raw_bits ? stq::launch_decode_raw(view(p), io, s0) : stq::launch_decode(view(p), io, s0);
    if (e == cudaSuccess && p->pivot_heads) e = stq::launch_decode_pivot_heads(view(p), io, s0);
    const cudaError_t eo = e == cudaSuccess && !direct ? cudaMemcpyAsync(y, d + L.y, vec, cudaMemcpyDeviceToHost, s0) : e;
    const cudaError_t er = cudaEventRecord(p->h_done, s0);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (eo != cudaSuccess) return cuda_fail(eo, "host-decode output copy");
    return er == cudaSuccess ? STQ_OK : cuda_fail(er, "host-decode event");
}

}  // namespace

extern "C" {

stq_status stq_decode_step_host(stq_pool *p, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, const float *q, const float *k, const float *v,
                                const float *beta, const float *gate, float *y, void *stream)
{
    stq_status st = check_launch_args(p, req_idx, slot_idx, n);
    if (st != STQ_OK) return st;
    if (n > 0 && (!q || !k || !v || !beta || !gate || !y))
        return fail(STQ_ERR_ARG, "a q/k/v/beta/gate/y pointer is NULL");
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_step_host");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    const cudaStream_t s0 = (cudaStream_t)stream;
    const HostLayout L = host_layout(p, n);
    cudaError_t e = host_staging(p, L.total, s0);
    if (e != cudaSuccess) return cuda_fail(e, "host-decode staging");
    e = join_async(p, s0);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    uint8_t *d = p->h_stage;
    const size_t vec = (size_t)n * p->H * kD * sizeof(float), per = (size_t)n * p->H * sizeof(float);
    const auto h2d = [&](size_t off, const void *src, size_t bytes) {
        return cudaMemcpyAsync(d + off, src, bytes, cudaMemcpyHostToDevice, s0);
    };
    p->h_used = true;
    e = h2d(L.req, req_idx, 4 * (size_t)n);
    if (e == cudaSuccess) e = h2d(L.slot, slot_idx, 4 * (size_t)n);
    if (e == cudaSuccess) e = h2d(L.q, q, vec);
    if (e == cudaSuccess) e = h2d(L.k, k, vec);
    if (e == cudaSuccess) e = h2d(L.v, v, vec);
    if (e == cudaSuccess) e = h2d(L.beta, beta, per);
    if (e == cudaSuccess) e = h2d(L.gate, gate, p->kind == STQ_KDA ? vec : per);
    if (e != cudaSuccess) {
        cudaEventRecord(p->h_done, s0);
        return cuda_fail(e, "host-decode input copy");
    }
    return host_decode_and_copy_out(p, n, L, y, s0);
}

stq_status stq_host_block_layout(const stq_pool *p, int32_t n, size_t offsets[7], size_t *bytes)
{
    if (p == nullptr || offsets == nullptr || bytes == nullptr) return fail(STQ_ERR_ARG, "NULL argument");
    if (n < 0) return fail(STQ_ERR_ARG, "n = %d", n);
    if ((long long)n * p->H > 0x7FFFFFFFll) return fail(STQ_ERR_ARG, "n * H too large");
    const HostLayout L = host_layout(p, n);
    const size_t o[7] = {L.req, L.slot, L.q, L.k, L.v, L.beta, L.gate};
    for (int a = 0; a < 7; ++a) offsets[a] = o[a];
    *bytes = L.inputs;
    return STQ_OK;
}

stq_status stq_decode_step_host_block(stq_pool *p, int32_t n, const void *block, size_t bytes, float *y,
                                      void *stream)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    if (n < 0) return fail(STQ_ERR_ARG, "n = %d", n);
    if ((long long)n * p->H > 0x7FFFFFFFll) return fail(STQ_ERR_ARG, "n * H too large");
    if (n > 0 && (block == nullptr || y == nullptr)) return fail(STQ_ERR_ARG, "block or y is NULL");
    const HostLayout L = host_layout(p, n);
    if (bytes != L.inputs)
        return fail(STQ_ERR_ARG, "block of %zu bytes; the layout for n = %d takes %zu", bytes, n, L.inputs);
    if (n == 0) return STQ_OK;
    if (fault("launch")) return fail(STQ_ERR_CUDA, "injected launch failure (STQ_FAULT=launch)");
    DeviceGuard g(p->device);
    NvtxRange nvtx("stq_decode_step_host_block");
    if (!g.ok) return fail(STQ_ERR_CUDA, "cannot select device %d", p->device);
    const cudaStream_t s0 = (cudaStream_t)stream;
    cudaError_t e = host_staging(p, L.total, s0);
    if (e != cudaSuccess) return cuda_fail(e, "host-decode staging");
    e = join_async(p, s0);
    if (e != cudaSuccess) return cuda_fail(e, "wait for the pending write-back");
    uint8_t *d = p->h_stage;
    p->h_used = true;
    e = cudaMemcpyAsync(d, block, L.inputs, cudaMemcpyHostToDevice, s0);
    if (e != cudaSuccess) {
        cudaEventRecord(p->h_done, s0);
        return cuda_fail(e, "host-decode input copy");
    }
    return host_decode_and_copy_out(p, n, L, y, s0);
}

stq_status stq_pool_join(stq_pool *p, void *stream)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    DeviceGuard g(p->device);
    cudaError_t e = join_async(p, (cudaStream_t)stream);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "wait for the pending write-back");
}

stq_status stq_export_slot(const stq_pool *p, int32_t req, int32_t slot, void *host_dst,
                           size_t bytes)
{
    if (p == nullptr || host_dst == nullptr) return fail(STQ_ERR_ARG, "NULL argument");
    if (req < 0 || req >= p->R || slot < 0 || slot >= p->S)
        return fail(STQ_ERR_ARG, "(request %d, slot %d) out of range", req, slot);
    if (bytes != p->slot_bytes)
        return fail(STQ_ERR_ARG, "bytes = %zu, slot holds %zu", bytes, p->slot_bytes);
    DeviceGuard g(p->device);
    const uint8_t *src = p->d_pages + ((size_t)req * p->S + slot) * p->slot_bytes;
    cudaError_t e = join_host(p);
    if (e == cudaSuccess) e = cudaMemcpy(host_dst, src, bytes, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "export");
}

stq_status stq_import_slot(stq_pool *p, int32_t req, int32_t slot, const void *host_src,
                           size_t bytes)
{
    if (p == nullptr || host_src == nullptr) return fail(STQ_ERR_ARG, "NULL argument");
    if (req < 0 || req >= p->R || slot < 0 || slot >= p->S)
        return fail(STQ_ERR_ARG, "(request %d, slot %d) out of range", req, slot);
    if (bytes != p->slot_bytes)
        return fail(STQ_ERR_ARG, "bytes = %zu, slot holds %zu", bytes, p->slot_bytes);
    DeviceGuard g(p->device);
    uint8_t *dst = p->d_pages + ((size_t)req * p->S + slot) * p->slot_bytes;
    cudaError_t e = join_host(p);
    if (e == cudaSuccess) e = cudaMemcpy(dst, host_src, bytes, cudaMemcpyHostToDevice);
    return e == cudaSuccess ? STQ_OK : cuda_fail(e, "import");
}

stq_status stq_pool_check(stq_pool *p, void *stream)
{
    if (p == nullptr) return fail(STQ_ERR_ARG, "pool is NULL");
    DeviceGuard g(p->device);
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = join_host(p);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    uint32_t word = 0;
    e = cudaMemcpy(&word, p->d_err, 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(p->d_err, 0, 4);
    if (e != cudaSuccess) return cuda_fail(e, "error word");
    if (word & stq::kErrTimeout) return fail(STQ_ERR_TIMEOUT, "a device-side wait timed out");
    if (word & stq::kErrIndex) return fail(STQ_ERR_INDEX, "request or slot index out of range");
    if (word & stq::kErrDuplicate) return fail(STQ_ERR_INDEX, "a (request, slot) pair named twice in one call");
    if (word & stq::kErrNonFinite) return fail(STQ_ERR_NONFINITE, "non-finite value in the step");
    return STQ_OK;
}

}  // extern "C"
