// stq_kernels.cu -- sm_100a quantize / dequantize kernels of the packed state pool.
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
// State Quantization" (paper.rainbus.top/paper/2609.38169).  Sections cited
// by name: "gated delta rule" (S_t = (I - b k k^T) D S_{t-1} + b k v^T),
// "PTQ" (Q(x) = s clip(round(x/s), -q_b, q_b)), "core method"
// (X^_ij = r_i c_j z_ij), "method steps" (online decode steps 1-7).
//
// Page layout (one (request, slot, head) tile): 128 fp32 row scales (or 128
// binary16 scales), then 128 rows of 128 b_i-bit two's complement codes
// (16 b_i bytes per row, little-endian bit order), padded to 128 bytes.  4- and
// 8-bit code j sits at bits [j b, (j + 1) b) of its row; 6-bit codes go in
// groups of eight, group g's 48 bits split into a 32-bit word at byte 4 g and a
// 16-bit half at byte 64 + 2 g.  A raw page is the row-major state itself in
// binary16 or fp32.
#include <cstdint>

#include <cuda_fp16.h>

#include "stq_internal.h"

namespace stq {
namespace {


__device__ __forceinline__ int qmax_of(int b) { return (1 << (b - 1)) - 1; }

// ---------------------------------------------------------------- quantize / dequantize

// Byte offset of row i and its width, from the per-head tables.
__device__ __forceinline__ uint8_t *tile_page(const PoolView &p, int req, int slot, int h)
{
    return p.pages + (static_cast<size_t>(req) * p.S + slot) * p.slot_bytes + p.t.head_off[h];
}

// fp32 state -> packed page: mu = fl32(S / (r c)) (fp64 quotient), s = fl32(max|mu| / q_b),
// z = clip(rint(fl32(mu / s)), -q_b, q_b).  A 16-bit row is an FP16 pivot: its scale
// slot holds 1 and it stores mu rounded once to binary16 (in a fitted page
// mu = fl32(S / r), without the column factor).  With fitted column factors the
// codes are taken with the table's c, then every column is refitted over the
// non-pivot rows in fp64, c_j = sum_i w_i^2 v_ij S_ij / sum_i w_i^2 v_ij^2 with
// v_ij = s_i r_i z_ij (each term formed in the oracle's operation order), and
// stored in the page.  One warp per row.
__global__ void __launch_bounds__(256) quantize_kernel(PoolView p, const int32_t *req_idx,
                                                       const int32_t *slot_idx, const float *state)
{
    __shared__ double fit_sum[8][2][kD];  // per-warp column sums of the fit (num, den)
    const int tile = blockIdx.x;
    const int ni = tile / p.H, h = tile - ni * p.H;
    const int req = req_idx[ni], slot = slot_idx[ni];
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    uint8_t *page = tile_page(p, req, slot, h);
    const float *S = state + static_cast<size_t>(tile) * kD * kD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4 c4 = *reinterpret_cast<const float4 *>(p.t.c + h * kD + lane * 4);
    const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
    const float *wrow = p.t.w + static_cast<size_t>(h) * kD;
    double fnum[4] = {0.0, 0.0, 0.0, 0.0}, fden[4] = {0.0, 0.0, 0.0, 0.0};
    bool bad = false;
    for (int i = warp; i < kD; i += 8) {
        const int b = p.t.row_bits[h * kD + i];
        const int qb = qmax_of(b);
        const double r = static_cast<double>(p.t.r[h * kD + i]);
        const float4 x4 = *reinterpret_cast<const float4 *>(S + i * kD + lane * 4);
        const float x[4] = {x4.x, x4.y, x4.z, x4.w};
        float mu[4];
        float a = 0.0f;
        const bool pivot_fit = b == 16 && p.fit;  // a fitted page's pivot row leaves c out
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            mu[t] = static_cast<float>(static_cast<double>(x[t]) / (pivot_fit ? r : r * static_cast<double>(cj[t])));
            a = fmaxf(a, fabsf(mu[t]));
            bad |= !isfinite(x[t]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (b == 16) {
            const __half2 h01 = __floats2half2_rn(mu[0], mu[1]), h23 = __floats2half2_rn(mu[2], mu[3]);
            uint2 w;
            w.x = *reinterpret_cast<const uint32_t *>(&h01);
            w.y = *reinterpret_cast<const uint32_t *>(&h23);
            *reinterpret_cast<uint2 *>(page + p.t.row_off[h * kD + i] + lane * 8) = w;
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            bad |= !(isfinite(f01.x) && isfinite(f01.y) && isfinite(f23.x) && isfinite(f23.y));
            if (lane == 0) {
                if (p.scale_bytes == 2) reinterpret_cast<__half *>(page)[i] = __float2half_rn(1.0f);
                else reinterpret_cast<float *>(page)[i] = 1.0f;
            }
            continue;
        }
        float s = __fdiv_rn(a, static_cast<float>(qb));
        __half s16 = __float2half_rn(s);
        if (p.scale_bytes == 2) s = __half2float(s16);  // the scale as stored
        bad |= !isfinite(s);
        uint32_t code[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            int zz = 0;
            if (s > 0.0f && isfinite(s)) {
                float rz = rintf(__fdiv_rn(mu[t], s));
                rz = fminf(fmaxf(rz, -static_cast<float>(qb)), static_cast<float>(qb));
                zz = static_cast<int>(rz);
            }
            code[t] = static_cast<uint32_t>(zz);
        }
        uint8_t *row = page + p.t.row_off[h * kD + i];
        if (b == 8) {
            *reinterpret_cast<uint32_t *>(row + lane * 4) = (code[0] & 255u) | (code[1] & 255u) << 8 |
                                                            (code[2] & 255u) << 16 | (code[3] & 255u) << 24;
        } else if (b == 4) {
            *reinterpret_cast<uint16_t *>(row + lane * 2) = static_cast<uint16_t>(
                (code[0] & 15u) | (code[1] & 15u) << 4 | (code[2] & 15u) << 8 | (code[3] & 15u) << 12);
        } else {
            // lanes 2g, 2g + 1 hold the 8 codes of group g: its 48-bit string is w(2g) | w(2g + 1) << 24
            const uint32_t w = (code[0] & 63u) | (code[1] & 63u) << 6 | (code[2] & 63u) << 12 | (code[3] & 63u) << 18;
            const uint32_t nb = __shfl_xor_sync(0xffffffffu, w, 1);
            if (lane & 1) *reinterpret_cast<uint16_t *>(row + 64 + (lane >> 1) * 2) = static_cast<uint16_t>(w >> 8);
            else *reinterpret_cast<uint32_t *>(row + (lane >> 1) * 4) = w | nb << 24;
        }
        if (lane == 0) {
            if (p.scale_bytes == 2) reinterpret_cast<__half *>(page)[i] = s16;
            else reinterpret_cast<float *>(page)[i] = s;
        }
        if (p.fit) {
            const double wi = static_cast<double>(wrow[i]);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const double v = static_cast<double>(s) * r * static_cast<double>(static_cast<int>(code[t]));
                fnum[t] += wi * wi * v * static_cast<double>(x[t]);
                fden[t] += wi * wi * v * v;
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, kErrNonFinite);
    if (p.fit) {  // uniform over the CTA
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            fit_sum[warp][0][lane * 4 + t] = fnum[t];
            fit_sum[warp][1][lane * 4 + t] = fden[t];
        }
        __syncthreads();
        if (threadIdx.x < kD) {
            const int j = threadIdx.x;
            double num = 0.0, den = 0.0;
            for (int w = 0; w < 8; ++w) {
                num += fit_sum[w][0][j];
                den += fit_sum[w][1][j];
            }
            const float cn = den > 0.0 ? static_cast<float>(num / den) : p.t.c[h * kD + j];
            if (!isfinite(cn)) atomicOr(p.err, kErrNonFinite);
            reinterpret_cast<float *>(page + p.scale_bytes * kD)[j] = cn;
        }
    }
}

// packed page -> fp32 reconstruction fl32(((s r) c) z) computed in fp64 (z: the binary16
// value of a pivot row, without c in a fitted page).  One warp per row.
__global__ void __launch_bounds__(256) dequantize_kernel(PoolView p, const int32_t *req_idx,
                                                         const int32_t *slot_idx, float *state)
{
    const int tile = blockIdx.x;
    const int ni = tile / p.H, h = tile - ni * p.H;
    const int req = req_idx[ni], slot = slot_idx[ni];
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    const uint8_t *page = tile_page(p, req, slot, h);
    float *S = state + static_cast<size_t>(tile) * kD * kD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the column factors: the page's own when they are fitted, else the table's
    const float4 c4 = *reinterpret_cast<const float4 *>((p.fit ? reinterpret_cast<const float *>(page + p.scale_bytes * kD)
                                                                : p.t.c + h * kD) + lane * 4);
    const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
    for (int i = warp; i < kD; i += 8) {
        const int b = p.t.row_bits[h * kD + i];
        const float sc = p.scale_bytes == 2 ? __half2float(reinterpret_cast<const __half *>(page)[i])
                                            : reinterpret_cast<const float *>(page)[i];
        const double sr = static_cast<double>(sc) * static_cast<double>(p.t.r[h * kD + i]);
        const uint8_t *row = page + p.t.row_off[h * kD + i];
        double zz[4];
        if (b == 16) {
            const uint2 w = *reinterpret_cast<const uint2 *>(row + lane * 8);
            const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
            const float2 c2 = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
            zz[0] = a.x;
            zz[1] = a.y;
            zz[2] = c2.x;
            zz[3] = c2.y;
        } else if (b == 8) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(row + lane * 4);
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (24 - 8 * t)) >> 24;
        } else if (b == 4) {
            const uint32_t w = *reinterpret_cast<const uint16_t *>(row + lane * 2);
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (28 - 4 * t)) >> 28;
        } else {
            const uint32_t lo = *reinterpret_cast<const uint32_t *>(row + (lane >> 1) * 4);
            const uint32_t hi = *reinterpret_cast<const uint16_t *>(row + 64 + (lane >> 1) * 2);
            const uint32_t w = (lane & 1) ? lo >> 24 | hi << 8 : lo & 0xFFFFFFu;
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (26 - 6 * t)) >> 26;
        }
        const bool pivot_fit = b == 16 && p.fit;  // a fitted page's pivot row leaves c out
        float4 o;
        o.x = static_cast<float>(sr * (pivot_fit ? 1.0 : static_cast<double>(cj[0])) * zz[0]);
        o.y = static_cast<float>(sr * (pivot_fit ? 1.0 : static_cast<double>(cj[1])) * zz[1]);
        o.z = static_cast<float>(sr * (pivot_fit ? 1.0 : static_cast<double>(cj[2])) * zz[2]);
        o.w = static_cast<float>(sr * (pivot_fit ? 1.0 : static_cast<double>(cj[3])) * zz[3]);
        *reinterpret_cast<float4 *>(S + i * kD + lane * 4) = o;
    }
}

// Raw pages: the state rounded once to binary16 (round to nearest even) or
// copied as fp32, and back.  256 threads, 4 consecutive elements each per step.
template <int BITS>
__global__ void __launch_bounds__(256) quantize_raw_kernel(PoolView p, const int32_t *req_idx,
                                                           const int32_t *slot_idx, const float *state)
{
    const int tile = blockIdx.x;
    const int ni = tile / p.H, h = tile - ni * p.H;
    const int req = req_idx[ni], slot = slot_idx[ni];
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    uint8_t *page = tile_page(p, req, slot, h);
    const float *S = state + static_cast<size_t>(tile) * kD * kD;
    bool bad = false;
    for (int e = threadIdx.x * 4; e < kD * kD; e += 256 * 4) {
        const float4 x = *reinterpret_cast<const float4 *>(S + e);
        if (BITS == 32) {
            *reinterpret_cast<float4 *>(page + 4 * e) = x;
            bad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
        } else {
            const __half2 a = __floats2half2_rn(x.x, x.y), b = __floats2half2_rn(x.z, x.w);
            uint2 w;
            w.x = *reinterpret_cast<const uint32_t *>(&a);
            w.y = *reinterpret_cast<const uint32_t *>(&b);
            *reinterpret_cast<uint2 *>(page + 2 * e) = w;
            const float2 fa = __half22float2(a), fb = __half22float2(b);
            bad |= !(isfinite(fa.x) && isfinite(fa.y) && isfinite(fb.x) && isfinite(fb.y));
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(p.err, kErrNonFinite);
}

template <int BITS>
__global__ void __launch_bounds__(256) dequantize_raw_kernel(PoolView p, const int32_t *req_idx,
                                                             const int32_t *slot_idx, float *state)
{
    const int tile = blockIdx.x;
    const int ni = tile / p.H, h = tile - ni * p.H;
    const int req = req_idx[ni], slot = slot_idx[ni];
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {
        if (threadIdx.x == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    const uint8_t *page = tile_page(p, req, slot, h);
    float *S = state + static_cast<size_t>(tile) * kD * kD;
    for (int e = threadIdx.x * 4; e < kD * kD; e += 256 * 4) {
        float4 x;
        if (BITS == 32) {
            x = *reinterpret_cast<const float4 *>(page + 4 * e);
        } else {
            const uint2 w = *reinterpret_cast<const uint2 *>(page + 2 * e);
            const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
            const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
            x = make_float4(a.x, a.y, b.x, b.y);
        }
        *reinterpret_cast<float4 *>(S + e) = x;
    }
}

// Debug check: entry e marks bit req * S + slot of `seen` (cleared before the
// launch); finding it already set means the pair is named twice.  Out-of-range
// pairs are left to the kernels that follow, which report them.
__global__ void __launch_bounds__(256) duplicate_kernel(const int32_t *req_idx, const int32_t *slot_idx, int n,
                                                        int R, int S, uint32_t *seen, uint32_t *err)
{
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const int r = req_idx[e], s = slot_idx[e];
    if (r < 0 || r >= R || s < 0 || s >= S) return;
    const uint32_t key = static_cast<uint32_t>(r) * static_cast<uint32_t>(S) + static_cast<uint32_t>(s);
    const uint32_t bit = 1u << (key & 31u);
    if (atomicOr(&seen[key >> 5], bit) & bit) atomicOr(err, kErrDuplicate);
}

}  // namespace

cudaError_t launch_duplicate_check(const int32_t *req_idx, const int32_t *slot_idx, int n, int R, int S,
                                   uint32_t *seen, uint32_t *err, cudaStream_t stream)
{
    const size_t words = (static_cast<size_t>(R) * S + 31) / 32;
    cudaError_t e = cudaMemsetAsync(seen, 0, words * sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    duplicate_kernel<<<(n + 255) / 256, 256, 0, stream>>>(req_idx, slot_idx, n, R, S, seen, err);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_quantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                            int n, const float *state, cudaStream_t stream)
{
    if (p.raw_bits == 32) quantize_raw_kernel<32><<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    else if (p.raw_bits == 16) quantize_raw_kernel<16><<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    else quantize_kernel<<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                              int n, float *state, cudaStream_t stream)
{
    if (p.raw_bits == 32) dequantize_raw_kernel<32><<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    else if (p.raw_bits == 16) dequantize_raw_kernel<16><<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    else dequantize_kernel<<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    count_launch();
    return cudaGetLastError();
}

}  // namespace stq
