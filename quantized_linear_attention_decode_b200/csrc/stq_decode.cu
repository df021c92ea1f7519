// stq_decode.cu -- the fused quantized decode step (sm_100a).
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
// State Quantization" (paper.rainbus.top/paper/2609.38169), online decode
// ("method steps", the paper's Table C2, steps 1-7) for Gated DeltaNet
// (D = alpha I) and Kimi Delta Attention (D = diag(d)) heads:
//   S^ = reconstruct(codes, scales)      X = D S^ + beta k (v^T - k^T D S^)
//   y  = X^T q (before requantisation)   codes, scales = quantize_rows(X)
//
// Design (B200): persistent CTAs, two per SM, 256 threads each.  A CTA walks
// its tiles (one (request, head) state each) in a fixed stride; thread 0
// keeps a four-stage ring of shared-memory buffers filled three tiles ahead
// with bulk async copies (packed page, q, k, v, r, c, row tables, KDA decay),
// completion tracked by one mbarrier per stage.  The requantised codes and
// scales go from registers straight to the page in global memory (coalesced
// per row).  Thread (rg, cg) owns rows [8 rg, 8 rg + 8)
// and columns [8 cg, 8 cg + 8) of the 128 x 128 tile in registers as
// floats.  With e_i = g_i s_i r_i (decayed row scale):
//   v_old_j = c_j sum_i (k_i e_i) z_ij        y_j = c_j sum_i (q_i e_i) z_ij + u_j (k.q)
//   u_j     = beta (v_j - v_old_j)            X_ij / c_j = e_i w_ij,  w_ij = z_ij + (k_i/e_i)(u_j/c_j)
//   s'_i    = |e_i| max_j |w_ij| / (r_i q_b)  z'_ij = round(w_ij q_b sign(e_i) / max_j |w_ij|)
// Codes become floats with the 2^23 trick (a byte or field OR-ed into the
// mantissa of 2^23, then 2^23 + 2^(b-1) subtracted), pairs of columns are
// processed with packed fma.rn.f32x2, and requantised codes are read back
// from the mantissa of fma(w, inv, 2^23 + 2^(b-1)).
#include <cstddef>
#include <cstdint>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int kThreads = 256;
constexpr int kStages = 4;
constexpr int kMaxPage = kScaleBytes + 16 * 8 * kD;    // 16896: every row at 8 bits
constexpr unsigned long long kWaitNs = 1000000000ull;  // bounded waits give up after 1 s

struct __align__(128) Stage {
    uint8_t page[kMaxPage];
    // the head's table block, one bulk copy (same layout as the pool's block)
    float r[kD], c[kD];
    uint16_t row_off[kD];
    uint8_t row_bits[kD];
    uint8_t pad[kHeadBlock - 4 * kD - 4 * kD - 2 * kD - kD];
    // per-tile vectors, stored from registers by all threads (prefetched two tiles ahead)
    float q[kD], k[kD], v[kD], g[kD];
};
static_assert(offsetof(Stage, q) - offsetof(Stage, r) == kHeadBlock, "head block layout");
static_assert(sizeof(Stage) % 128 == 0, "stage size");

// Per-tile row data, double buffered by tile parity: written while the
// previous tile finishes, read by both passes of the tile.
struct __align__(16) RowCoef {
    float4 kl[kD];     // {k_i e_i, k_i e_i, q_i e_i, q_i e_i}
    float h[kD];       // k_i / e_i, or k_i for a dropped row
    float mrq[kD];     // e_i / (r_i q_b(i)) (1 / (r_i q_b) for a dropped row): s'_i = |mrq_i| max_j |w_ij|
    uint16_t off[kD];  // byte offset of row i inside the page
    uint8_t bits[kD];
    uint32_t deg[4];   // bit i: row i's old content is dropped (e_i = 0)
    uint8_t *page;     // the tile's page in global memory
    float kq;
    uint32_t valid;
};

struct __align__(128) Smem {
    Stage st[kStages];
    RowCoef rc[2];
    float red[2048];   // column partial sums [8 warps][v, y][128]
    float ut[kD];      // u_j / c_j
    uint8_t *stage_page[kStages];
    uint32_t stage_valid[kStages];
    float beta[kStages], alpha[kStages];
    uint32_t raw[8][4];  // {req, slot, head offset, page bytes} of tile k in raw[k % 8]
    uint32_t flags;
    unsigned long long full[kStages];
};

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

__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity)
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

__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          unsigned long long *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// small asynchronous copies global -> shared, completed per thread with cp.async.wait_group
__device__ __forceinline__ void cp_async4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// packed pair arithmetic (sm_100: one instruction for two fp32 lanes)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// approximate reciprocal (one MUFU op; relative error below 2^-22 for normal inputs)
__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float f_of(uint32_t u) { return __uint_as_float(u); }

// ---------------------------------------------------------------- codecs
//
// unpack: the 8 codes of columns [8 cg, 8 cg + 8) of one packed row (in
// shared memory) as float pairs (first pass).  The b-bit two's complement code z becomes
// the offset code u = z + 2^(b-1) (one XOR per word), u is placed in the
// mantissa of 2^23 (exact: 2^23 + u) and 2^23 + 2^(b-1) is subtracted
// (exact).
//
// Requantised codes come back as the bit patterns of fl(w inv + kMagicOut):
// 2^23 + u for 4 and 6 bits, 1.5 * 2^23 + z for 8 bits (packed by Chunk<B>).

template <int B> struct Codec;

template <> struct Codec<8> {
    static constexpr float kMagicOut = 12582912.0f;  // 1.5 * 2^23: low byte = z (two's complement)
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        const uint2 w = *reinterpret_cast<const uint2 *>(rowp + cg * 8);
        const uint32_t x0 = w.x ^ 0x80808080u, x1 = w.y ^ 0x80808080u;
        const float2 off = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
        z[0] = fadd2(make_float2(f_of(__byte_perm(x0, 0x4B000000u, 0x7650)), f_of(__byte_perm(x0, 0x4B000000u, 0x7651))), off);
        z[1] = fadd2(make_float2(f_of(__byte_perm(x0, 0x4B000000u, 0x7652)), f_of(__byte_perm(x0, 0x4B000000u, 0x7653))), off);
        z[2] = fadd2(make_float2(f_of(__byte_perm(x1, 0x4B000000u, 0x7650)), f_of(__byte_perm(x1, 0x4B000000u, 0x7651))), off);
        z[3] = fadd2(make_float2(f_of(__byte_perm(x1, 0x4B000000u, 0x7652)), f_of(__byte_perm(x1, 0x4B000000u, 0x7653))), off);
    }
};

template <> struct Codec<4> {
    static constexpr float kMagicOut = 8388616.0f;  // 2^23 + 8: mantissa = u = z + 8 in [1, 15]
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        const uint32_t x = *reinterpret_cast<const uint32_t *>(rowp + cg * 4) ^ 0x88888888u;
        const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
        const float2 off = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
        z[0] = fadd2(make_float2(f_of(__byte_perm(lo, 0x4B000000u, 0x7650)), f_of(__byte_perm(hi, 0x4B000000u, 0x7650))), off);
        z[1] = fadd2(make_float2(f_of(__byte_perm(lo, 0x4B000000u, 0x7651)), f_of(__byte_perm(hi, 0x4B000000u, 0x7651))), off);
        z[2] = fadd2(make_float2(f_of(__byte_perm(lo, 0x4B000000u, 0x7652)), f_of(__byte_perm(hi, 0x4B000000u, 0x7652))), off);
        z[3] = fadd2(make_float2(f_of(__byte_perm(lo, 0x4B000000u, 0x7653)), f_of(__byte_perm(hi, 0x4B000000u, 0x7653))), off);
    }
};

template <> struct Codec<6> {
    static constexpr float kMagicOut = 8388640.0f;  // 2^23 + 32: mantissa = u = z + 32 in [1, 63]
    __device__ __forceinline__ static uint32_t field(uint32_t a)
    {
        return ((a ^ 0x20u) & 0x3Fu) | 0x4B000000u;
    }
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        // 8 codes = 6 bytes at offset 6 cg (2-byte aligned): read the two aligned words around them
        const uint32_t base = (cg >> 1) * 12 + (cg & 1) * 4;
        const uint32_t sh = (cg & 1) * 16;
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(rowp + base);
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(rowp + base + 4);
        const uint32_t lo = __funnelshift_r(w0, w1, sh);
        const uint32_t hi = w1 >> sh;
        const float2 off = make_float2(-8388640.0f, -8388640.0f);  // -(2^23 + 32)
        z[0] = fadd2(make_float2(f_of(field(lo)), f_of(field(lo >> 6))), off);
        z[1] = fadd2(make_float2(f_of(field(lo >> 12)), f_of(field(lo >> 18))), off);
        z[2] = fadd2(make_float2(f_of(field(lo >> 24)), f_of(field(__funnelshift_r(lo, hi, 30)))), off);
        z[3] = fadd2(make_float2(f_of(field(hi >> 4)), f_of(field(hi >> 10))), off);
    }
};

__device__ __forceinline__ void unpack_any(int b, const uint8_t *rowp, int cg, float2 z[4])
{
    if (b == 8) Codec<8>::unpack(rowp, cg, z);
    else if (b == 6) Codec<6>::unpack(rowp, cg, z);
    else Codec<4>::unpack(rowp, cg, z);
}

__device__ __forceinline__ float magic_out(int b)
{
    return b == 8 ? Codec<8>::kMagicOut : (b == 6 ? Codec<6>::kMagicOut : Codec<4>::kMagicOut);
}


// ---------------------------------------------------------------- 32-code chunks
//
// The second pass gives each row to a quad of lanes: lane q of the quad owns
// columns [32 q, 32 q + 32), i.e. the chunk of 4 b bytes at row offset 4 b q.

template <int B> struct Chunk;

template <> struct Chunk<8> {
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int q, float2 z[16])
    {
        const uint4 a = *reinterpret_cast<const uint4 *>(rowp + 32 * q);
        const uint4 b = *reinterpret_cast<const uint4 *>(rowp + 32 * q + 16);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        const float2 off = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t x = w[k] ^ 0x80808080u;
            z[2 * k] = fadd2(make_float2(f_of(__byte_perm(x, 0x4B000000u, 0x7650)), f_of(__byte_perm(x, 0x4B000000u, 0x7651))), off);
            z[2 * k + 1] = fadd2(make_float2(f_of(__byte_perm(x, 0x4B000000u, 0x7652)), f_of(__byte_perm(x, 0x4B000000u, 0x7653))), off);
        }
    }
    __device__ __forceinline__ static void store(uint8_t *rowg, int q, const uint32_t b[32])
    {
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            w[k] = __byte_perm(__byte_perm(b[4 * k], b[4 * k + 1], 0x0040), __byte_perm(b[4 * k + 2], b[4 * k + 3], 0x0040), 0x5410);
        *reinterpret_cast<uint4 *>(rowg + 32 * q) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(rowg + 32 * q + 16) = make_uint4(w[4], w[5], w[6], w[7]);
    }
};

template <> struct Chunk<4> {
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int q, float2 z[16])
    {
        const uint4 a = *reinterpret_cast<const uint4 *>(rowp + 16 * q);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        const float2 off = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t x = w[k] ^ 0x88888888u;
            const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int t = 0; t < 4; ++t)
                z[4 * k + t] = fadd2(make_float2(f_of(__byte_perm(lo, 0x4B000000u, 0x7650 + t)),
                                                 f_of(__byte_perm(hi, 0x4B000000u, 0x7650 + t))), off);
        }
    }
    __device__ __forceinline__ static void store(uint8_t *rowg, int q, const uint32_t b[32])
    {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t acc = b[8 * k];
#pragma unroll
            for (int t = 1; t < 8; ++t) acc += b[8 * k + t] << (4 * t);
            w[k] = (acc - 0xFB000000u) ^ 0x88888888u;
        }
        *reinterpret_cast<uint4 *>(rowg + 16 * q) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <> struct Chunk<6> {
    __device__ __forceinline__ static void group(uint32_t lo, uint32_t hi, float2 z[4])
    {
        const float2 off = make_float2(-8388640.0f, -8388640.0f);  // -(2^23 + 32)
        z[0] = fadd2(make_float2(f_of(Codec<6>::field(lo)), f_of(Codec<6>::field(lo >> 6))), off);
        z[1] = fadd2(make_float2(f_of(Codec<6>::field(lo >> 12)), f_of(Codec<6>::field(lo >> 18))), off);
        z[2] = fadd2(make_float2(f_of(Codec<6>::field(lo >> 24)), f_of(Codec<6>::field(__funnelshift_r(lo, hi, 30)))), off);
        z[3] = fadd2(make_float2(f_of(Codec<6>::field(hi >> 4)), f_of(Codec<6>::field(hi >> 10))), off);
    }
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int q, float2 z[16])
    {
        const uint2 a = *reinterpret_cast<const uint2 *>(rowp + 24 * q);
        const uint2 b = *reinterpret_cast<const uint2 *>(rowp + 24 * q + 8);
        const uint2 c = *reinterpret_cast<const uint2 *>(rowp + 24 * q + 16);
        group(a.x, a.y, z);
        group(__funnelshift_r(a.y, b.x, 16), b.x >> 16, z + 4);
        group(b.y, c.x, z + 8);
        group(__funnelshift_r(c.x, c.y, 16), c.y >> 16, z + 12);
    }
    // 8 codes (b[t] = 0x4B000000 + u_t) -> 48 bits: lo (32) and hi (low 16 of the result)
    __device__ __forceinline__ static void pack8(const uint32_t *b, uint32_t &lo, uint32_t &hi)
    {
        lo = b[0] + (b[1] << 6) + (b[2] << 12) + (b[3] << 18) + (b[4] << 24) + (b[5] << 30);
        lo = (lo - 0x0B000000u) ^ 0x20820820u;
        hi = ((b[5] >> 2) + (b[6] << 4) + (b[7] << 10)) ^ 0x8208u;
    }
    __device__ __forceinline__ static void store(uint8_t *rowg, int q, const uint32_t b[32])
    {
        uint32_t l0, h0, l1, h1, l2, h2, l3, h3;
        pack8(b, l0, h0);
        pack8(b + 8, l1, h1);
        pack8(b + 16, l2, h2);
        pack8(b + 24, l3, h3);
        uint2 *dst = reinterpret_cast<uint2 *>(rowg + 24 * q);
        dst[0] = make_uint2(l0, __byte_perm(h0, l1, 0x5410));
        dst[1] = make_uint2(__byte_perm(l1, h1, 0x5432), l2);
        dst[2] = make_uint2(__byte_perm(h2, l3, 0x5410), __byte_perm(l3, h3, 0x5432));
    }
};

// ---------------------------------------------------------------- one tile
//
// Pass 1: thread (rg, cg) = (2 warp + lane / 16, lane % 16) reads rows
// [8 rg, 8 rg + 8) x columns [8 cg, 8 cg + 8), accumulates the two column
// sums and leaves per-warp partials in red.  B = 4, 6, 8: every row has B
// bits (GDN); B = 0: per-row widths (KDA).
template <int B>
__device__ __forceinline__ void pass1(Smem &sm, const Stage &S, const RowCoef &R)
{
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int rgl = lane >> 4, cg = lane & 15;
    const int i0 = (warp * 2 + rgl) * 8;
    float2 av[4], ay[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) av[p] = ay[p] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        float2 z[4];
        if (B != 0) Codec<B == 0 ? 8 : B>::unpack(S.page + kScaleBytes + 16 * B * i, cg, z);
        else unpack_any(R.bits[i], S.page + R.off[i], cg, z);
        const float4 kl = R.kl[i];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            av[p] = ffma2(make_float2(kl.x, kl.y), z[p], av[p]);
            ay[p] = ffma2(make_float2(kl.z, kl.w), z[p], ay[p]);
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        av[p].x += __shfl_xor_sync(0xffffffffu, av[p].x, 16);
        av[p].y += __shfl_xor_sync(0xffffffffu, av[p].y, 16);
        ay[p].x += __shfl_xor_sync(0xffffffffu, ay[p].x, 16);
        ay[p].y += __shfl_xor_sync(0xffffffffu, ay[p].y, 16);
    }
    // half 0 keeps the v-sums, half 1 the y-sums; column j of a sum sits at
    // ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3) (conflict-free 16-byte stores)
    const float2 *src = rgl == 0 ? av : ay;
    float *dst = &sm.red[warp * 256 + rgl * 128 + cg * 4];
    *reinterpret_cast<float4 *>(dst) = make_float4(src[0].x, src[0].y, src[1].x, src[1].y);
    *reinterpret_cast<float4 *>(dst + 64) = make_float4(src[2].x, src[2].y, src[3].x, src[3].y);
}

// Per column (threads 0..127): v_old, u, y, u / c.
__device__ __forceinline__ void column_epilogue(Smem &sm, const Stage &S, const RowCoef &R,
                                                const DecodeIO &io, int tile, float beta)
{
    const int j = threadIdx.x;
    const int at = ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3);
    float vz = 0.0f, yz = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        vz += sm.red[w * 256 + at];
        yz += sm.red[w * 256 + 128 + at];
    }
    const float cj = S.c[j];
    const float u = beta * (S.v[j] - cj * vz);
    const float yj = fmaf(u, R.kq, cj * yz);
    io.y[static_cast<size_t>(tile) * kD + j] = yj;
    sm.ut[j] = u * rcp_approx(cj);
    if (!isfinite(u) || !isfinite(yj)) atomicOr(&sm.flags, kErrNonFinite);
}

// Per row (threads 128..255) of the next tile: decayed scale e_i and the
// coefficients both passes need; warp 4 also forms k.q.
template <int KIND>
__device__ __forceinline__ void row_setup(Smem &sm, const Stage &S, RowCoef &R, int s)
{
    const int r = threadIdx.x - kD;
    const bool valid = sm.stage_valid[s] != 0;
    if (r == 0) {
        R.page = sm.stage_page[s];
        R.valid = valid;
    }
    if (!valid) return;
    const float sc = reinterpret_cast<const float *>(S.page)[r];
    const float g = KIND == STQ_GDN ? sm.alpha[s] : S.g[r];
    const float rr = S.r[r];
    const float e = (g * sc) * rr;
    const float kr = S.k[r];
    const float ka = kr * e, la = S.q[r] * e;
    const float hq = kr * rcp_approx(e);
    const bool dropped = !(e != 0.0f && fabsf(hq) <= 1e30f);
    const int b = S.row_bits[r];
    const float rq = rr * static_cast<float>((1 << (b - 1)) - 1);
    R.kl[r] = make_float4(ka, ka, la, la);
    R.h[r] = dropped ? kr : hq;
    R.mrq[r] = __fdiv_rn(dropped ? 1.0f : e, rq);
    R.off[r] = S.row_off[r];
    R.bits[r] = static_cast<uint8_t>(b);
    const uint32_t bal = __ballot_sync(0xffffffffu, dropped);
    if ((r & 31) == 0) R.deg[r >> 5] = bal;
    if (!isfinite(e)) atomicOr(&sm.flags, kErrNonFinite);
    if (r < 32) {
        const float4 k4 = *reinterpret_cast<const float4 *>(&S.k[r * 4]);
        const float4 q4 = *reinterpret_cast<const float4 *>(&S.q[r * 4]);
        float a = k4.x * q4.x;
        a = fmaf(k4.y, q4.y, a);
        a = fmaf(k4.z, q4.z, a);
        a = fmaf(k4.w, q4.w, a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (r == 0) R.kq = a;
    }
}

// Pass 2: quad q = lane % 4 of row i owns columns [32 q, 32 q + 32); each
// thread takes rows rp and rp + 64 (rp = tid / 4).  Re-reads the old codes,
// w = z + h u~, row absmax (local, then two shuffles), new scale, requantise,
// store 4 b bytes of codes per row (and lane 0 the scale) to global memory.
template <int B>
__device__ __forceinline__ void pass2_row(Smem &sm, const Stage &S, const RowCoef &R, int i, int q,
                                          const float2 ut2[16])
{
    const int b = B != 0 ? B : R.bits[i];
    const bool dropped = (R.deg[i >> 5] >> (i & 31)) & 1u;
    const float hq = R.h[i];
    const float2 h2 = make_float2(hq, hq);
    float2 w[16];
    if (!dropped) {
        const uint8_t *rowp = S.page + (B != 0 ? kScaleBytes + 16 * B * i : R.off[i]);
        if (B != 0) Chunk<B == 0 ? 8 : B>::unpack(rowp, q, w);
        else if (b == 8) Chunk<8>::unpack(rowp, q, w);
        else if (b == 6) Chunk<6>::unpack(rowp, q, w);
        else Chunk<4>::unpack(rowp, q, w);
#pragma unroll
        for (int p = 0; p < 16; ++p) w[p] = ffma2(h2, ut2[p], w[p]);
    } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) w[p] = fmul2(h2, ut2[p]);
    }
    float m = fmaxf(fabsf(w[0].x), fabsf(w[0].y));
#pragma unroll
    for (int p = 1; p < 16; ++p) m = max3(m, fabsf(w[p].x), fabsf(w[p].y));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    const float qb = static_cast<float>((1 << (b - 1)) - 1);
    const float mrq = R.mrq[i];
    float inv = 0.0f, snew = 0.0f;
    if (m >= 1e-30f && m <= 3.0e38f) {
        inv = copysignf(qb * rcp_approx(m), mrq);
        snew = fabsf(mrq) * m;
    } else if (m > 0.0f && m < 1e-30f) {
        inv = copysignf(__fdiv_rn(qb, m), mrq);
        snew = fabsf(mrq) * m;
    } else if (!(m == 0.0f)) {
        atomicOr(&sm.flags, kErrNonFinite);
    }
    uint8_t *page = R.page;
    if (q == 0) reinterpret_cast<float *>(page)[i] = snew;
    const float mg = B != 0 ? Codec<B == 0 ? 8 : B>::kMagicOut : magic_out(b);
    const float2 inv2 = make_float2(inv, inv), mg2 = make_float2(mg, mg);
    uint32_t bits[32];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const float2 t = ffma2(w[p], inv2, mg2);
        bits[2 * p] = __float_as_uint(t.x);
        bits[2 * p + 1] = __float_as_uint(t.y);
    }
    uint8_t *rowg = page + (B != 0 ? kScaleBytes + 16 * B * i : R.off[i]);
    if (B != 0) Chunk<B == 0 ? 8 : B>::store(rowg, q, bits);
    else if (b == 8) Chunk<8>::store(rowg, q, bits);
    else if (b == 6) Chunk<6>::store(rowg, q, bits);
    else Chunk<4>::store(rowg, q, bits);
}

template <int B>
__device__ __forceinline__ void pass2(Smem &sm, const Stage &S, const RowCoef &R)
{
    const int tid = threadIdx.x;
    const int q = tid & 3, rp = tid >> 2;
    float2 ut2[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(&sm.ut[32 * q + 4 * k]);
        ut2[2 * k] = make_float2(a.x, a.y);
        ut2[2 * k + 1] = make_float2(a.z, a.w);
    }
    pass2_row<B>(sm, S, R, rp, q, ut2);
    pass2_row<B>(sm, S, R, rp + 64, q, ut2);
}

// ---------------------------------------------------------------- kernel

// Where a tile's page lives.
struct TileRaw {
    int req, slot, h;
    uint32_t hoff, bytes;
};

struct TileRef {
    uint8_t *page;
    uint32_t bytes;
    int h;
    bool valid;
};

__device__ __forceinline__ TileRaw load_raw(const PoolView &p, const DecodeIO &io, int tile)
{
    TileRaw t;
    const int ni = tile / p.H;
    t.h = tile - ni * p.H;
    t.req = io.req_idx[ni];
    t.slot = io.slot_idx[ni];
    t.hoff = p.t.head_off[t.h];
    t.bytes = p.t.page_bytes[t.h];
    return t;
}

__device__ __forceinline__ TileRef resolve(const PoolView &p, const TileRaw &r)
{
    TileRef t;
    t.h = r.h;
    t.valid = r.req >= 0 && r.req < p.R && r.slot >= 0 && r.slot < p.S;
    t.page = t.valid ? p.pages + (static_cast<size_t>(r.req) * p.S + r.slot) * p.slot_bytes + r.hoff : nullptr;
    t.bytes = t.valid ? r.bytes : 0u;
    return t;
}

template <int KIND>
__device__ __forceinline__ void issue(Smem &sm, int s, const PoolView &p, const TileRef &t)
{
    Stage &S = sm.st[s];
    sm.stage_page[s] = t.page;
    sm.stage_valid[s] = t.valid;
    if (!t.valid) {
        atomicOr(&sm.flags, kErrIndex);
        mbar_arrive(&sm.full[s]);  // completes the phase with no data; the tile is skipped
        return;
    }
    mbar_arrive_expect_tx(&sm.full[s], t.bytes + kHeadBlock);
    bulk_load(S.page, t.page, t.bytes, &sm.full[s]);
    bulk_load(S.r, p.t.block + static_cast<size_t>(t.h) * kHeadBlock, kHeadBlock, &sm.full[s]);
}

// Asynchronous prefetch, one cp.async group per thread per tile (issued after
// the first barrier of tile i, waited with wait_group 1 before the first
// barrier of tile i + 2): q, k, v (and the KDA decay), beta, alpha of tile
// i + 3 into its stage, and the raw location {req, slot, head offset, page
// bytes} of tile i + 5.
template <int KIND>
__device__ __forceinline__ void prefetch(Smem &sm, const PoolView &p, const DecodeIO &io, int i, int t3, int t5,
                                         int tiles)
{
    const int t = threadIdx.x;
    if (t3 < tiles) {
        Stage &S = sm.st[(i + 3) % kStages];
        const size_t base = static_cast<size_t>(t3) * kD + 4 * (t & 31);
        if (t < 32) cp_async16(&S.q[4 * t], io.q + base);
        else if (t < 64) cp_async16(&S.k[4 * (t - 32)], io.k + base);
        else if (t < 96) cp_async16(&S.v[4 * (t - 64)], io.v + base);
        else if (t < 128) {
            if (KIND == STQ_KDA) cp_async16(&S.g[4 * (t - 96)], io.gate + base);
        } else if (t == 128) {
            cp_async4(&sm.beta[(i + 3) % kStages], io.beta + t3);
        } else if (t == 129) {
            if (KIND == STQ_GDN) cp_async4(&sm.alpha[(i + 3) % kStages], io.gate + t3);
        }
    }
    if (t5 < tiles && t >= 130 && t < 134) {
        const int ni = t5 / p.H, h = t5 - ni * p.H;
        uint32_t *dst = &sm.raw[(i + 5) & 7][t - 130];
        if (t == 130) cp_async4(dst, io.req_idx + ni);
        else if (t == 131) cp_async4(dst, io.slot_idx + ni);
        else if (t == 132) cp_async4(dst, p.t.head_off + h);
        else cp_async4(dst, p.t.page_bytes + h);
    }
    cp_async_commit();
}

// Synchronous fill of a stage's vectors and beta/alpha (first tiles only).
template <int KIND>
__device__ __forceinline__ void fill_sync(Smem &sm, const DecodeIO &io, int s, int tile)
{
    const int t = threadIdx.x;
    Stage &S = sm.st[s];
    const size_t base = static_cast<size_t>(tile) * kD;
    if (t < kD) {
        S.q[t] = io.q[base + t];
        S.k[t] = io.k[base + t];
    } else {
        S.v[t - kD] = io.v[base + t - kD];
        if (KIND == STQ_KDA) S.g[t - kD] = io.gate[base + t - kD];
    }
    if (t == 0) {
        sm.beta[s] = io.beta[tile];
        sm.alpha[s] = KIND == STQ_GDN ? io.gate[tile] : 0.0f;
    }
}

__device__ __forceinline__ TileRaw raw_from_smem(const Smem &sm, const PoolView &p, int tile, int k)
{
    TileRaw r;
    const int ni = tile / p.H;
    r.h = tile - ni * p.H;
    r.req = static_cast<int>(sm.raw[k & 7][0]);
    r.slot = static_cast<int>(sm.raw[k & 7][1]);
    r.hoff = sm.raw[k & 7][2];
    r.bytes = sm.raw[k & 7][3];
    return r;
}

// Persistent CTA: tiles first, first + G, first + 2G, ... (G = gridDim.x).
// Per tile i (stage i % 4, row data rc[i % 2]):
//   all:       pass 1 of tile i                                        | barrier
//   thread 0:  issue tile i + 3 (page and head block) into the stage of tile i - 1
//   all:       cp.async prefetch of tile i + 3's vectors, tile i + 5's location
//   warps 0-3: column epilogue of tile i (y, u / c)
//   warps 4-7: wait for tile i + 1's stage, its row coefficients       | barrier
//   all:       pass 2 of tile i (re-reads the codes; new codes and scales to global memory)
// A stage is last read by pass 2 of its tile, which every warp finishes
// before the first barrier of the next tile.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(PoolView p, DecodeIO io, int tiles)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    const int first = blockIdx.x;
    if (first >= tiles) return;

    if (tid == 0) {
        sm.flags = 0;
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
        for (int a = 0; a < 3; ++a) {
            const int t = first + a * G;
            if (t < tiles) issue<KIND>(sm, a, p, resolve(p, load_raw(p, io, t)));
        }
        for (int a = 3; a < 5; ++a) {
            const int t = first + a * G;
            if (t < tiles) {
                const TileRaw r = load_raw(p, io, t);
                sm.raw[a][0] = static_cast<uint32_t>(r.req);
                sm.raw[a][1] = static_cast<uint32_t>(r.slot);
                sm.raw[a][2] = r.hoff;
                sm.raw[a][3] = r.bytes;
            }
        }
    }
    for (int a = 0; a < 3; ++a)
        if (first + a * G < tiles) fill_sync<KIND>(sm, io, a, first + a * G);
    __syncthreads();
    bool timed_out = false;
    if (tid >= kD) {
        if (mbar_wait_bounded(&sm.full[0], 0)) row_setup<KIND>(sm, sm.st[0], sm.rc[0], 0);
        else timed_out = true;
    }
    timed_out = __syncthreads_or(timed_out) != 0;

    int i = 0;
    for (int tile = first; tile < tiles && !timed_out; tile += G, ++i) {
        const int s = i % kStages;
        const RowCoef &R = sm.rc[i & 1];
        const Stage &S = sm.st[s];
        const bool valid = R.valid != 0;
        const int b = valid ? R.bits[0] : 8;
        if (valid) {
            if (KIND == STQ_KDA) pass1<0>(sm, S, R);
            else if (b == 8) pass1<8>(sm, S, R);
            else if (b == 6) pass1<6>(sm, S, R);
            else pass1<4>(sm, S, R);
        }
        cp_async_wait<1>();
        __syncthreads();
        if (tid == 0 && tile + 3 * G < tiles)
            issue<KIND>(sm, (i + 3) % kStages, p, resolve(p, raw_from_smem(sm, p, tile + 3 * G, i + 3)));
        prefetch<KIND>(sm, p, io, i, tile + 3 * G, tile + 5 * G, tiles);
        bool tout = false;
        if (tid < kD) {
            if (valid) column_epilogue(sm, S, R, io, tile, sm.beta[s]);
        } else if (tile + G < tiles) {
            const int sn = (i + 1) % kStages;
            if (mbar_wait_bounded(&sm.full[sn], ((i + 1) / kStages) & 1)) row_setup<KIND>(sm, sm.st[sn], sm.rc[(i + 1) & 1], sn);
            else tout = true;
        }
        timed_out = __syncthreads_or(tout) != 0;
        if (valid) {
            if (KIND == STQ_KDA) pass2<0>(sm, S, R);
            else if (b == 8) pass2<8>(sm, S, R);
            else if (b == 6) pass2<6>(sm, S, R);
            else pass2<4>(sm, S, R);
        }
    }
    cp_async_wait<0>();  // no copy may land in this CTA's shared memory after it exits

    __syncthreads();  // every warp's flags are in before thread 0 reads them
    if (tid == 0) {
        if (timed_out) {
            // a stage never arrived: report, then wait (bounded) for the loads still in flight
            // (tiles i, i + 1, i + 2 of this CTA, counted after the loop's last increment)
            atomicOr(p.err, kErrTimeout);
            for (int k = i; k < i + 3; ++k) {
                const int t = first + k * G;
                if (t < tiles) mbar_wait_bounded(&sm.full[k % kStages], (k / kStages) & 1);
            }
        }
        if (sm.flags) atomicOr(p.err, sm.flags);
    }
}

constexpr int kMaxDevices = 64;

template <int KIND>
cudaError_t launch(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    // per device: SM count, and the dynamic shared-memory opt-in of this kernel
    static int sms[kMaxDevices] = {0};
    const int smem = static_cast<int>(sizeof(Smem));
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (sms[dev] == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(decode_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        sms[dev] = n > 0 ? n : 148;
    }
    const int tiles = io.n * p.H;
    const int grid = tiles < 2 * sms[dev] ? tiles : 2 * sms[dev];
    decode_kernel<KIND><<<grid, kThreads, smem, stream>>>(p, io, tiles);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return p.kind == STQ_KDA ? launch<STQ_KDA>(p, io, stream) : launch<STQ_GDN>(p, io, stream);
}

}  // namespace stq
