// stq_internal.h -- shared between the host side (stq_api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "stq.h"

namespace stq {

constexpr int kD = 128;            // d_k = d_v
constexpr int kScaleBytes = 4 * kD; // fp32 scales at the start of a page
constexpr int kPageAlign = 128;    // pages are padded to this many bytes
constexpr int kMaxStagedPage = kScaleBytes + 4 * kD + 16 * 8 * kD;  // largest page the fused kernel stages
                                                                    // (8 bits per row, fitted column factors)
constexpr size_t kStaticScratchFloats = size_t(1) << 20;  // built-in u~ buffer: 4 MiB, 8192 tiles

// device error word bits
constexpr uint32_t kErrIndex = 1u;
constexpr uint32_t kErrNonFinite = 2u;
constexpr uint32_t kErrTimeout = 4u;
constexpr uint32_t kErrDuplicate = 8u;  // a (request, slot) pair named twice in one call (debug checks)

// Per-head tables, one device allocation:
//   head_off[H]    byte offset of the head's page inside a slot
//   page_bytes[H]  size of the head's page
//   row_off[H][128] byte offset of row i inside the page (scales come first)
//   row_bits[H][128]
//   r[H][128], c[H][128]
//   w[H][128]       row weights of the column fit
//   block[H][kHeadBlock]: r, c, 1 / (r q_b), row_off, row_bits, decode row order of one head
//                  side by side, so that the decode kernel fetches them with one copy
constexpr int kHeadBlock = 2048;  // 512 (r) + 512 (c) + 512 (1 / (r q_b)) + 256 (row_off) + 128 (row_bits) + 128 (row order)
constexpr int kFitBytes = 4 * kD;  // a fitted page's own column factors (fp32), after the scales
struct Tables {
    const uint32_t *head_off;
    const uint32_t *page_bytes;
    const uint16_t *row_off;
    const uint8_t *row_bits;
    const float *r;
    const float *c;
    const float *w;
    const uint8_t *block;
    const int32_t *pivot_head;  // GDN: the FP16 pivot heads, ascending (n_pivot_heads of them)
};

struct PoolView {
    uint8_t *pages;      // [R][S][slot_bytes]
    size_t slot_bytes;
    int R, S, H;
    int kind;
    int scale_bytes;     // bytes per row scale: 4 (fp32) or 2 (binary16); 0 in a raw pool
    int raw_bits;        // 16 or 32 in a raw pool (every unit), else 0
    int pivots;          // nonzero if 16-bit (FP16 pivot) units sit among quantized ones
    int fit;             // nonzero: pages carry column factors refitted at every quantisation
    int per_row;         // KDA: some head has a pass warp whose 16 rows the width-specialised
                         // passes cannot take, so every tile takes the per-row path
    int n_pivot_heads;   // GDN: heads held in FP16 (their own kernel), listed in t.pivot_head
    Tables t;
    uint32_t *err;
    unsigned long long wait_ns;  // limit of every bounded device-side wait
    uint32_t stall_tx;           // test hook: bytes the first stage of CTA 0 expects beyond its copies
};

struct DecodeIO {
    const int32_t *req_idx;
    const int32_t *slot_idx;
    int n;
    const float *q, *k, *v, *beta, *gate;  // the write-back reads u~ through v (q, beta unused)
    float *y;
    float *u_out;  // the readout's u~ = u / c per tile [n][H][128]; unused by the other modes
};

cudaError_t launch_decode(const PoolView &p, const DecodeIO &io, cudaStream_t stream);
cudaError_t launch_decode_raw(const PoolView &p, const DecodeIO &io, cudaStream_t stream);
// GDN FP16 pivot heads of a quantized pool (pages larger than kMaxStagedPage), one CTA per tile
cudaError_t launch_decode_pivot_heads(const PoolView &p, const DecodeIO &io, cudaStream_t stream);
cudaError_t launch_decode_readout(const PoolView &p, const DecodeIO &io, cudaStream_t stream);
cudaError_t launch_decode_writeback(const PoolView &p, const DecodeIO &io, cudaStream_t stream);
// Marks the call's (request, slot) pairs in `seen` (R * S bits, cleared first on
// the stream) and sets kErrDuplicate in `err` for a pair named twice.
cudaError_t launch_duplicate_check(const int32_t *req_idx, const int32_t *slot_idx, int n, int R, int S,
                                   uint32_t *seen, uint32_t *err, cudaStream_t stream);
cudaError_t launch_quantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                            int n, const float *state, cudaStream_t stream);
cudaError_t launch_dequantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                              int n, float *state, cudaStream_t stream);

void count_launch();

// Records a printf-style message for stq_last_error() and returns st.
stq_status fail_status(stq_status st, const char *fmt, ...);

}  // namespace stq
