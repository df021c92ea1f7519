// stq_kernels.cu -- sm_100a kernels of the quantized gated delta-rule decode.
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
// State Quantization" (paper.rainbus.top/paper/2609.38169).  Sections cited
// by name: "gated delta rule" (S_t = (I - b k k^T) D S_{t-1} + b k v^T),
// "PTQ" (Q(x) = s clip(round(x/s), -q_b, q_b)), "core method"
// (X^_ij = r_i c_j z_ij), "method steps" (online decode steps 1-7).
//
// Page layout (one (request, slot, head) tile): 128 fp32 row scales, then
// 128 rows of 128 b_i-bit two's complement codes (16 b_i bytes per row,
// little-endian bit order), padded to 128 bytes.
#include <cstdint>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int kThreads = 256;                   // 8 warps per tile
constexpr int kMaxPage = kScaleBytes + 16 * 8 * kD;  // 16896 bytes (all rows 8-bit)
constexpr unsigned long long kWaitNs = 1000000000ull;  // bounded waits give up after 1 s

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of the barrier; gives up after kWaitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}

// bulk async copy global -> shared, completion signalled on the barrier
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// bulk async copy shared -> global (bulk group)
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the async (bulk copy) proxy
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ int qmax_of(int b) { return (1 << (b - 1)) - 1; }

// ---------------------------------------------------------------- code I/O

// The 8 codes of columns [8 cg, 8 cg + 8) of one packed row, as floats.
__device__ __forceinline__ void unpack8(const uint8_t *rowp, int b, int cg, float z[8])
{
    if (b == 8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(rowp + cg * 8);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            z[t] = static_cast<float>(static_cast<int>(w.x << (24 - 8 * t)) >> 24);
            z[4 + t] = static_cast<float>(static_cast<int>(w.y << (24 - 8 * t)) >> 24);
        }
    } else if (b == 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(rowp + cg * 4);
#pragma unroll
        for (int t = 0; t < 8; ++t) z[t] = static_cast<float>(static_cast<int>(w << (28 - 4 * t)) >> 28);
    } else {  // 6 bits: 8 codes = 6 bytes at a 2-byte aligned offset
        const uint32_t off = cg * 6, base = off & ~3u, sh = (off & 3u) * 8u;
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(rowp + base);
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(rowp + base + 4);
        const uint32_t lo = __funnelshift_r(w0, w1, sh);
        const uint32_t hi = w1 >> sh;
        const uint64_t x = (static_cast<uint64_t>(hi) << 32) | lo;
#pragma unroll
        for (int t = 0; t < 8; ++t)
            z[t] = static_cast<float>(static_cast<int>(static_cast<int64_t>(x << (58 - 6 * t)) >> 58));
    }
}

// Store 8 codes (low b bits of each word, two's complement) at columns [8 cg, 8 cg + 8).
__device__ __forceinline__ void pack8(uint8_t *rowp, int b, int cg, const uint32_t c[8])
{
    if (b == 8) {
        uint2 w;
        w.x = (c[0] & 255u) | (c[1] & 255u) << 8 | (c[2] & 255u) << 16 | (c[3] & 255u) << 24;
        w.y = (c[4] & 255u) | (c[5] & 255u) << 8 | (c[6] & 255u) << 16 | (c[7] & 255u) << 24;
        *reinterpret_cast<uint2 *>(rowp + cg * 8) = w;
    } else if (b == 4) {
        uint32_t w = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) w |= (c[t] & 15u) << (4 * t);
        *reinterpret_cast<uint32_t *>(rowp + cg * 4) = w;
    } else {
        uint64_t x = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) x |= static_cast<uint64_t>(c[t] & 63u) << (6 * t);
        uint16_t *p = reinterpret_cast<uint16_t *>(rowp + cg * 6);
        p[0] = static_cast<uint16_t>(x);
        p[1] = static_cast<uint16_t>(x >> 16);
        p[2] = static_cast<uint16_t>(x >> 32);
    }
}

// ---------------------------------------------------------------- decode step

struct __align__(128) DecodeSmem {
    uint8_t page[kMaxPage];
    float red[kThreads / 32][2][kD];  // per-warp column partial sums
    float k[kD], q[kD], v[kD], g[kD];
    float r[kD], c[kD];
    float kap[kD], lam[kD];  // per-row coefficients of the two column sums
    float hh[kD], m[kD];     // per-row split of the updated row: t = m (z + hh u~)
    float ut[kD];            // u_j / c_j
    float sinv[kD];          // per-row quantisation multiplier
    uint16_t row_off[kD];
    uint8_t row_bits[kD];
    uint8_t deg[kD];         // rows whose old content is dropped (e == 0)
    float kq;
    uint32_t flags;
    uint64_t bar;
};

// One CTA per (entry, head) tile.  Thread (rg, cg) owns rows [8 rg, 8 rg + 8)
// and columns [8 cg, 8 cg + 8) of the 128 x 128 state.
//
// With e_i = g_i s_i r_i (decayed row scale) and z the old codes:
//   P_ij      = e_i c_j z_ij                       (D S^, "method steps" 1-2)
//   v_old_j   = c_j sum_i (k_i e_i) z_ij
//   u_j       = beta (v_j - v_old_j)
//   y_j       = c_j sum_i (q_i e_i) z_ij + u_j (k . q)  (= X^T q, step 3)
//   X_ij / c_j = e_i (z_ij + (k_i / e_i) (u_j / c_j)) = m_i w_ij
// and the row's new absmax scale and codes follow from w alone:
//   s'_i = |m_i| max_j |w_ij| / (r_i q_b),  z'_ij = round(w_ij q_b sign(m_i) / max_j |w_ij|).
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(PoolView p, DecodeIO io)
{
    __shared__ DecodeSmem sm;
    const int tid = threadIdx.x;
    const int tile = blockIdx.x;
    const int ni = tile / p.H;
    const int h = tile - ni * p.H;
    const int req = io.req_idx[ni];
    const int slot = io.slot_idx[ni];
    if (req < 0 || req >= p.R || slot < 0 || slot >= p.S) {
        if (tid == 0) atomicOr(p.err, kErrIndex);
        return;
    }
    uint8_t *page_g = p.pages + (static_cast<size_t>(req) * p.S + slot) * p.slot_bytes + p.t.head_off[h];
    const uint32_t pbytes = p.t.page_bytes[h];

    if (tid == 0) {
        sm.flags = 0;
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&sm.bar, pbytes);
        bulk_load(sm.page, page_g, pbytes, &sm.bar);
    }
    const size_t vec = static_cast<size_t>(tile) * kD;
    const float beta = io.beta[tile];
    if (tid < kD) {
        sm.k[tid] = io.k[vec + tid];
        sm.q[tid] = io.q[vec + tid];
        sm.r[tid] = p.t.r[h * kD + tid];
        sm.row_off[tid] = p.t.row_off[h * kD + tid];
        sm.row_bits[tid] = p.t.row_bits[h * kD + tid];
    } else {
        const int j = tid - kD;
        sm.v[j] = io.v[vec + j];
        sm.g[j] = p.kind == STQ_KDA ? io.gate[vec + j] : io.gate[tile];
        sm.c[j] = p.t.c[h * kD + j];
    }
    __syncthreads();
    if (!mbar_wait_bounded(&sm.bar, 0)) {
        // the page never arrived: report, wait (bounded) for the copy, leave the tile as it was
        if (tid == 0) atomicOr(p.err, kErrTimeout);
        mbar_wait_bounded(&sm.bar, 0);
        return;
    }

    // ---- per-row coefficients (threads 0..127) and k.q (warp 4)
    if (tid < kD) {
        const int i = tid;
        const float s = reinterpret_cast<const float *>(sm.page)[i];
        const float e = (sm.g[i] * s) * sm.r[i];
        const float ki = sm.k[i];
        sm.kap[i] = ki * e;
        sm.lam[i] = sm.q[i] * e;
        const float hq = ki / e;
        const bool degenerate = !(e != 0.0f && fabsf(hq) <= 1e30f);
        sm.deg[i] = degenerate;
        sm.hh[i] = degenerate ? ki : hq;
        sm.m[i] = degenerate ? 1.0f : e;
        if (!isfinite(e)) atomicOr(&sm.flags, kErrNonFinite);
    } else if (tid < kD + 32) {
        const int lane = tid - kD;
        float a = 0.0f;
#pragma unroll
        for (int t = 0; t < 4; ++t) a = fmaf(sm.k[lane * 4 + t], sm.q[lane * 4 + t], a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) sm.kq = a;
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int rg = warp * 2 + (lane >> 4), cg = lane & 15;
    const int i0 = rg * 8;

    // ---- pass 1: unpack the old codes, two column sums
    float z[8][8];
    float av[8], ay[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) av[jj] = ay[jj] = 0.0f;
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        unpack8(sm.page + sm.row_off[i], sm.row_bits[i], cg, z[ii]);
        const float ka = sm.kap[i], la = sm.lam[i];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            av[jj] = fmaf(ka, z[ii][jj], av[jj]);
            ay[jj] = fmaf(la, z[ii][jj], ay[jj]);
        }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        av[jj] += __shfl_xor_sync(0xffffffffu, av[jj], 16);
        ay[jj] += __shfl_xor_sync(0xffffffffu, ay[jj], 16);
    }
    if (lane < 16) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) sm.red[warp][0][cg * 8 + jj] = av[jj];
    } else {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) sm.red[warp][1][cg * 8 + jj] = ay[jj];
    }
    __syncthreads();

    // ---- per-column: v_old, u, y (threads 0..127)
    if (tid < kD) {
        const int j = tid;
        float vz = 0.0f, yz = 0.0f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            vz += sm.red[w][0][j];
            yz += sm.red[w][1][j];
        }
        const float cj = sm.c[j];
        const float vold = cj * vz;
        const float u = beta * (sm.v[j] - vold);
        const float yj = fmaf(u, sm.kq, cj * yz);
        io.y[vec + j] = yj;
        sm.ut[j] = u / cj;
        if (!isfinite(u) || !isfinite(yj)) atomicOr(&sm.flags, kErrNonFinite);
    }
    __syncthreads();

    // ---- pass 2: updated row values w, row absmax
    float ut[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) ut[jj] = sm.ut[cg * 8 + jj];
    float mx[8];
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        const float hq = sm.hh[i];
        float a = 0.0f;
        if (!sm.deg[i]) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                z[ii][jj] = fmaf(hq, ut[jj], z[ii][jj]);
                a = fmaxf(a, fabsf(z[ii][jj]));
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                z[ii][jj] = hq * ut[jj];
                a = fmaxf(a, fabsf(z[ii][jj]));
            }
        }
        mx[ii] = a;
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1)
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) mx[ii] = fmaxf(mx[ii], __shfl_xor_sync(0xffffffffu, mx[ii], o));

    // ---- per-row new scale and multiplier: lane cg < 8 of each half-warp takes row i0 + cg
    if (cg < 8) {
        float M = mx[0];
#pragma unroll
        for (int ii = 1; ii < 8; ++ii)
            if (cg == ii) M = mx[ii];
        const int i = i0 + cg;
        const int qb = qmax_of(sm.row_bits[i]);
        const float mi = sm.m[i];
        float inv = 0.0f, snew = 0.0f;
        if (M > 0.0f && M <= 3.0e38f) {
            inv = copysignf(static_cast<float>(qb) / M, mi);
            snew = (fabsf(mi) * M) / (sm.r[i] * static_cast<float>(qb));
        } else if (!(M == 0.0f)) {
            atomicOr(&sm.flags, kErrNonFinite);
        }
        sm.sinv[i] = inv;
        reinterpret_cast<float *>(sm.page)[i] = snew;
    }
    __syncwarp();

    // ---- requantise and pack in place: z' = round(w * inv) via the 1.5 * 2^23 rounding constant
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        const float inv = sm.sinv[i];
        uint32_t cw[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) cw[jj] = __float_as_uint(fmaf(z[ii][jj], inv, 12582912.0f));
        pack8(sm.page + sm.row_off[i], sm.row_bits[i], cg, cw);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(page_g, sm.page, pbytes);
        bulk_commit();
        if (sm.flags) atomicOr(p.err, sm.flags);
        bulk_wait_all();
    }
}

// ---------------------------------------------------------------- quantize / dequantize

// Byte offset of row i and its width, from the per-head tables.
__device__ __forceinline__ uint8_t *tile_page(const PoolView &p, int req, int slot, int h)
{
    return p.pages + (static_cast<size_t>(req) * p.S + slot) * p.slot_bytes + p.t.head_off[h];
}

// fp32 state -> packed page: mu = fl32(S / (r c)) (fp64 quotient), s = fl32(max|mu| / q_b),
// z = clip(rint(fl32(mu / s)), -q_b, q_b).  One warp per row.
__global__ void __launch_bounds__(256) quantize_kernel(PoolView p, const int32_t *req_idx,
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
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4 c4 = *reinterpret_cast<const float4 *>(p.t.c + h * kD + lane * 4);
    const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
    bool bad = false;
    for (int i = warp; i < kD; i += 8) {
        const int b = p.t.row_bits[h * kD + i];
        const int qb = qmax_of(b);
        const double r = static_cast<double>(p.t.r[h * kD + i]);
        const float4 x4 = *reinterpret_cast<const float4 *>(S + i * kD + lane * 4);
        const float x[4] = {x4.x, x4.y, x4.z, x4.w};
        float mu[4];
        float a = 0.0f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            mu[t] = static_cast<float>(static_cast<double>(x[t]) / (r * static_cast<double>(cj[t])));
            a = fmaxf(a, fabsf(mu[t]));
            bad |= !isfinite(x[t]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float s = __fdiv_rn(a, static_cast<float>(qb));
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
            const uint32_t w = (code[0] & 63u) | (code[1] & 63u) << 6 | (code[2] & 63u) << 12 | (code[3] & 63u) << 18;
            row[lane * 3 + 0] = static_cast<uint8_t>(w);
            row[lane * 3 + 1] = static_cast<uint8_t>(w >> 8);
            row[lane * 3 + 2] = static_cast<uint8_t>(w >> 16);
        }
        if (lane == 0) reinterpret_cast<float *>(page)[i] = s;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, kErrNonFinite);
}

// packed page -> fp32 reconstruction fl32(((s r) c) z) computed in fp64.  One warp per row.
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
    const float4 c4 = *reinterpret_cast<const float4 *>(p.t.c + h * kD + lane * 4);
    const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
    for (int i = warp; i < kD; i += 8) {
        const int b = p.t.row_bits[h * kD + i];
        const double sr = static_cast<double>(reinterpret_cast<const float *>(page)[i]) *
                          static_cast<double>(p.t.r[h * kD + i]);
        const uint8_t *row = page + p.t.row_off[h * kD + i];
        int zz[4];
        if (b == 8) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(row + lane * 4);
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (24 - 8 * t)) >> 24;
        } else if (b == 4) {
            const uint32_t w = *reinterpret_cast<const uint16_t *>(row + lane * 2);
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (28 - 4 * t)) >> 28;
        } else {
            const uint32_t w = row[lane * 3] | row[lane * 3 + 1] << 8 | row[lane * 3 + 2] << 16;
#pragma unroll
            for (int t = 0; t < 4; ++t) zz[t] = static_cast<int>(w << (26 - 6 * t)) >> 26;
        }
        float4 o;
        o.x = static_cast<float>(sr * static_cast<double>(cj[0]) * static_cast<double>(zz[0]));
        o.y = static_cast<float>(sr * static_cast<double>(cj[1]) * static_cast<double>(zz[1]));
        o.z = static_cast<float>(sr * static_cast<double>(cj[2]) * static_cast<double>(zz[2]));
        o.w = static_cast<float>(sr * static_cast<double>(cj[3]) * static_cast<double>(zz[3]));
        *reinterpret_cast<float4 *>(S + i * kD + lane * 4) = o;
    }
}

}  // namespace

cudaError_t launch_decode(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    const int tiles = io.n * p.H;
    decode_kernel<<<tiles, kThreads, 0, stream>>>(p, io);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_quantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                            int n, const float *state, cudaStream_t stream)
{
    quantize_kernel<<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const PoolView &p, const int32_t *req_idx, const int32_t *slot_idx,
                              int n, float *state, cudaStream_t stream)
{
    dequantize_kernel<<<n * p.H, 256, 0, stream>>>(p, req_idx, slot_idx, state);
    count_launch();
    return cudaGetLastError();
}

}  // namespace stq
