// stq_decode_raw.cu -- sm_100a decode step over raw (unquantized) state pages.
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
// State Quantization" (paper.rainbus.top/paper/2609.38169).  The same
// recurrence as the quantized step ("gated delta rule"; "method steps",
// steps 2-3) on a state stored as values: binary16 (the page's FP16 storage
// of pivot units, here for a whole pool) or fp32 (the unquantized control
// its state-update timings compare against):
//   P = D S,  u = beta (v - P^T k),  X = P + k u^T,  y = X^T q,  S <- round(X).
// y = P^T q + (k.q) u, so one pass over S forms both column sums.
//
// The same kernel advances the GDN FP16 pivot heads of a quantized pool
// (PIVOT): their page keeps the pool's scale section (slots of 1; in a fitted
// pool also its column factor section, unused) and stores mu = X / (r c) in
// binary16 (mu = X / r in a fitted pool: c_j = 1 below), so with P = g S and
// S_ij = r_i c_j mu_ij
//   column sums over (g k r)_i mu_ij and (g q r)_i mu_ij, times c_j;
//   mu'_ij = g mu_ij + (k_i / r_i) (u_j / c_j).
// CTAs of the other heads return at once.
//
// One CTA (256 threads) per (request, head) tile.  Thread (rg, cg) = (2 warp +
// lane / 16, lane % 16) holds rows [8 rg, 8 rg + 8) x columns [8 cg, 8 cg + 8)
// in registers between the two passes; a half-warp reads or writes one row's
// 128 contiguous values, so every access is a full 16-byte vector.  The kernel
// streams 2 x 32 KiB (binary16) or 2 x 64 KiB (fp32) per tile: HBM-bound.
#include <cstddef>
#include <cstdint>

#include <cuda_fp16.h>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int kRawThreads = 256;

__device__ __forceinline__ float2 ffma2r(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fmul2r(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 8 values of one row at columns [8 cg, 8 cg + 8): load (streaming) and store
template <int BITS> struct RawRow;

template <> struct RawRow<32> {
    __device__ __forceinline__ static void load(const uint8_t *row, int cg, float2 x[4])
    {
        const float4 *p = reinterpret_cast<const float4 *>(row) + 2 * cg;
        const float4 a = __ldcs(p), b = __ldcs(p + 1);
        x[0] = make_float2(a.x, a.y);
        x[1] = make_float2(a.z, a.w);
        x[2] = make_float2(b.x, b.y);
        x[3] = make_float2(b.z, b.w);
    }
    __device__ __forceinline__ static bool store(uint8_t *row, int cg, const float2 x[4])
    {
        float4 *p = reinterpret_cast<float4 *>(row) + 2 * cg;
        __stcs(p, make_float4(x[0].x, x[0].y, x[1].x, x[1].y));
        __stcs(p + 1, make_float4(x[2].x, x[2].y, x[3].x, x[3].y));
        bool ok = true;
#pragma unroll
        for (int t = 0; t < 4; ++t) ok &= isfinite(x[t].x) && isfinite(x[t].y);
        return ok;
    }
};

template <> struct RawRow<16> {
    __device__ __forceinline__ static void load(const uint8_t *row, int cg, float2 x[4])
    {
        const uint4 w = __ldcs(reinterpret_cast<const uint4 *>(row) + cg);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) x[t] = __half22float2(*reinterpret_cast<const __half2 *>(&u[t]));
    }
    __device__ __forceinline__ static bool store(uint8_t *row, int cg, const float2 x[4])
    {
        uint32_t u[4];
        bool ok = true;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const __half2 h = __float22half2_rn(x[t]);  // round to nearest even
            u[t] = *reinterpret_cast<const uint32_t *>(&h);
            const float2 back = __half22float2(h);
            ok &= isfinite(back.x) && isfinite(back.y);
        }
        __stcs(reinterpret_cast<uint4 *>(row) + cg, make_uint4(u[0], u[1], u[2], u[3]));
        return ok;
    }
};

template <int KIND, int BITS, bool PIVOT>
__global__ void __launch_bounds__(kRawThreads, 2) decode_raw_kernel(PoolView p, DecodeIO io)
{
    __shared__ __align__(16) float red[kRawThreads / 32][2][kD];  // column partials per warp
    __shared__ __align__(16) float gk[kD], gq[kD];                 // g_i k_i, g_i q_i
    __shared__ __align__(16) float ks[kD], us[kD];                 // k_i, u_j
    __shared__ float kqp[4];
    __shared__ uint32_t bad;

    // raw pools: block = tile; pivot heads: block = (entry, k-th pivot head)
    int ni, h;
    if (PIVOT) {
        ni = blockIdx.x / p.n_pivot_heads;
        h = p.t.pivot_head[blockIdx.x - ni * p.n_pivot_heads];
    } else {
        ni = blockIdx.x / p.H;
        h = blockIdx.x - ni * p.H;
    }
    const int tile = ni * p.H + h;
    if (PIVOT && p.t.row_bits[h * kD] != 16) return;  // a quantized head: the fused kernel's
    const int req = io.req_idx[ni], slot = io.slot_idx[ni];
    const int tid = threadIdx.x;
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {  // uniform over the CTA
        if (tid == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    uint8_t *page = p.pages + (static_cast<size_t>(req) * p.S + slot) * p.slot_bytes + p.t.head_off[h] +
                    (PIVOT ? p.scale_bytes * kD + (p.fit ? kFitBytes : 0) : 0);
    const size_t vec = static_cast<size_t>(tile) * kD;
    const int warp = tid >> 5, lane = tid & 31;
    const int rgl = lane >> 4, cg = lane & 15;
    const int i0 = (warp * 2 + rgl) * 8;
    constexpr int kRowBytes = kD * BITS / 8;

    // the state loads go first: 8 rows x 8 columns per thread, all in flight together
    float2 x[8][4];
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) RawRow<BITS>::load(page + (i0 + ii) * kRowBytes, cg, x[ii]);

    if (tid == 0) bad = 0;
    if (tid >= kD) {
        // rows: g_i k_i, g_i q_i, k_i, and the k.q partial of this warp
        const int r = tid - kD;
        const float g = KIND == STQ_GDN ? io.gate[tile] : io.gate[vec + r];
        const float k = io.k[vec + r], q = io.q[vec + r];
        const float rr = PIVOT ? p.t.r[h * kD + r] : 1.0f;
        gk[r] = PIVOT ? (g * k) * rr : g * k;
        gq[r] = PIVOT ? (g * q) * rr : g * q;
        ks[r] = PIVOT ? __fdiv_rn(k, rr) : k;
        float a = k * q;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if ((r & 31) == 0) kqp[r >> 5] = a;
    }
    __syncthreads();

    // pass 1: column sums of (g k)_i S_ij and (g q)_i S_ij
    float2 av[4], ay[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) av[t] = ay[t] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const float a = gk[i0 + ii], b = gq[i0 + ii];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            av[t] = ffma2r(make_float2(a, a), x[ii][t], av[t]);
            ay[t] = ffma2r(make_float2(b, b), x[ii][t], ay[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        av[t].x += __shfl_xor_sync(0xffffffffu, av[t].x, 16);
        av[t].y += __shfl_xor_sync(0xffffffffu, av[t].y, 16);
        ay[t].x += __shfl_xor_sync(0xffffffffu, ay[t].x, 16);
        ay[t].y += __shfl_xor_sync(0xffffffffu, ay[t].y, 16);
    }
    {
        const float2 *src = rgl == 0 ? av : ay;
        float4 *dst = reinterpret_cast<float4 *>(&red[warp][rgl][cg * 8]);
        dst[0] = make_float4(src[0].x, src[0].y, src[1].x, src[1].y);
        dst[1] = make_float4(src[2].x, src[2].y, src[3].x, src[3].y);
    }
    __syncthreads();

    // column epilogue: u_j = beta (v_j - (P^T k)_j), y_j = (P^T q)_j + (k.q) u_j
    if (tid < kD) {
        const int j = tid;
        float vz = 0.0f, yz = 0.0f;
#pragma unroll
        for (int w = 0; w < kRawThreads / 32; ++w) {
            vz += red[w][0][j];
            yz += red[w][1][j];
        }
        const float kq = (kqp[0] + kqp[1]) + (kqp[2] + kqp[3]);
        const float cj = PIVOT && !p.fit ? p.t.c[h * kD + j] : 1.0f;  // a fitted page's pivots leave c out
        const float u = io.beta[tile] * (io.v[vec + j] - (PIVOT ? cj * vz : vz));
        const float yj = fmaf(kq, u, PIVOT ? cj * yz : yz);
        io.y[vec + j] = yj;
        us[j] = PIVOT ? __fdiv_rn(u, cj) : u;
        if (!isfinite(u) || !isfinite(yj)) atomicOr(&bad, 1u);
    }
    __syncthreads();

    // pass 2: X = g S + k u^T, rounded once into the page
    float2 u2[4];
    {
        const float4 a = *reinterpret_cast<const float4 *>(&us[cg * 8]);
        const float4 b = *reinterpret_cast<const float4 *>(&us[cg * 8 + 4]);
        u2[0] = make_float2(a.x, a.y);
        u2[1] = make_float2(a.z, a.w);
        u2[2] = make_float2(b.x, b.y);
        u2[3] = make_float2(b.z, b.w);
    }
    const float gd = KIND == STQ_GDN ? io.gate[tile] : 0.0f;
    bool ok = true;
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        const float g = KIND == STQ_GDN ? gd : io.gate[vec + i];
        const float k = ks[i];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            x[ii][t] = ffma2r(make_float2(k, k), u2[t], fmul2r(make_float2(g, g), x[ii][t]));
        ok &= RawRow<BITS>::store(page + i * kRowBytes, cg, x[ii]);
    }
    if (!ok) atomicOr(&bad, 1u);
    __syncthreads();
    if (tid == 0 && bad) atomicOr(p.err, kErrNonFinite);
}

template <int KIND, int BITS, bool PIVOT = false>
cudaError_t launch_raw(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    const int blocks = io.n * (PIVOT ? p.n_pivot_heads : p.H);
    if (blocks == 0) return cudaSuccess;
    decode_raw_kernel<KIND, BITS, PIVOT><<<blocks, kRawThreads, 0, stream>>>(p, io);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_pivot_heads(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return launch_raw<STQ_GDN, 16, true>(p, io, stream);
}

cudaError_t launch_decode_raw(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    if (p.raw_bits == 16)
        return p.kind == STQ_KDA ? launch_raw<STQ_KDA, 16>(p, io, stream) : launch_raw<STQ_GDN, 16>(p, io, stream);
    return p.kind == STQ_KDA ? launch_raw<STQ_KDA, 32>(p, io, stream) : launch_raw<STQ_GDN, 32>(p, io, stream);
}

}  // namespace stq
