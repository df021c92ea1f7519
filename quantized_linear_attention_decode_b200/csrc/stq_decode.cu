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
// its tiles (one (request, head) state each) in a fixed stride; thread 96
// keeps a four-stage ring of shared-memory buffers filled three tiles ahead
// with bulk async copies (the packed page and the head's table block: r, c,
// row offsets, widths and order), completion tracked by one mbarrier per
// stage; q, k, v (and the KDA decay), beta and alpha come in by cp.async,
// also three tiles ahead.  The requantised codes and
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
// from the mantissa of fma(w, inv, M_b) (M_b = 2^23 + 2^(b-1) at 4 and 6
// bits, 1.5 * 2^23 at 8 bits).
//
// The same kernel, instantiated per mode, also runs the step split in two
// ("method steps", steps 3-7: the readout first, the requantisation and
// write-back on a separate stream): kReadout stops after the column epilogue
// and stores u~ = u / c per tile; kWriteback re-reads the page, takes u~ from
// that buffer in place of the column sums, and runs pass 2.  Both halves do
// the fused kernel's arithmetic, so the split step's y, codes and scales are
// bit-identical to the fused step's.
#include <cstddef>
#include <cstdint>

#include <cuda_fp16.h>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int kThreads = 256;

// kernel modes
constexpr int kFused = 0;      // the whole step (one state traversal)
constexpr int kReadout = 1;    // steps 1-3: y and u~; the page is only read
constexpr int kWriteback = 2;  // steps 4-7 given u~: requantise and pack in place
constexpr int kStages = 4;
constexpr int kRedStride = 288;  // floats per warp in red: 256 column partials, or the padded row-max exchange
constexpr int kMaxPage = kMaxStagedPage;               // 17408: every row at 8 bits, with fitted factors

struct __align__(128) Stage {
    uint8_t page[kMaxPage];
    // the head's table block, one bulk copy (same layout as the pool's block)
    float r[kD], c[kD];
    float inv_rq[kD];  // 1 / (r_i q_b(i))
    uint16_t row_off[kD];
    uint8_t row_bits[kD];
    uint8_t perm[kD];  // KDA: the row taken at each position (rows grouped by width)
    // per-tile vectors, stored from registers by all threads (prefetched two tiles ahead)
    float q[kD], k[kD], v[kD], g[kD];
};
static_assert(offsetof(Stage, q) - offsetof(Stage, r) == kHeadBlock, "head block layout");
static_assert(sizeof(Stage) % 128 == 0, "stage size");

// Per-tile row data, double buffered by tile parity: written while the
// previous tile finishes, read by both passes of the tile.  Indexed by
// position: thread (warp w, half g) takes positions 8 (2 w + g) .. + 7.  GDN
// position i is row i; a KDA head takes its rows in the order of its
// table's permutation, which groups rows of one width, so that the two
// halves of a warp mostly unpack and pack rows of the same width together.
struct __align__(16) RowCoef {
    float4 kl[kD];     // {k_i e_i, k_i e_i, q_i e_i, q_i e_i}
    float h[kD];       // k_i / e_i, or k_i for a dropped row
    float mrq[kD];     // e_i / (r_i q_b(i)) (1 / (r_i q_b) for a dropped row): s'_i = |mrq_i| max_j |w_ij|
    uint16_t off[kD];  // byte offset of row i inside the page
    uint8_t bits[kD];
    uint8_t row[kD];   // the row at each position
    uint8_t wbits[8];  // KDA: the width all 16 positions of pass warp w share, else 0
    float fb[kD];      // column fit: (w_i r_i)^2
    uint32_t deg[4];   // bit i: row i's old content is dropped (e_i = 0)
    uint8_t *page;     // the tile's page in global memory
    float kqp[4];      // k.q, partial sums of rows [32 w, 32 w + 32)
    uint32_t valid;
};

struct __align__(128) Smem {
    Stage st[kStages];
    RowCoef rc[2];
    float red[8 * kRedStride];  // per warp: column partial sums [v, y][128]; then row-max partials
    float rowinv[kD];  // per-row quantisation multiplier (pass 2)
    float red2[2048];  // column fit partial sums [8 warps][num, den][128], finished in the next tile
    float rowA[kD], rowB[kD];  // column fit row coefficients of pass 2: A = fa s', B = fb s'^2
    float fitc[kD];    // the column factors the tile's codes were taken with
    float ut[kD];      // u_j / c_j, column j at ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3)
    uint8_t *stage_page[kStages];
    const float *stage_w[kStages];  // the tile's head row weights (column fit)
    uint32_t stage_valid[kStages];
    float beta[kStages], alpha[kStages];
    uint32_t raw[8][5];  // {req, slot, head offset, page bytes, head} of tile k in raw[k % 8]
    uint32_t flags;
    uint32_t stop;     // a row-setup wait gave up (set by warps 4-7, read by all after a barrier)
    unsigned long long full[kStages];
    uint8_t *fit_page[2];    // page of the tile whose fit is pending, by tile parity
    uint32_t fit_pending[2];
};
// arrays read or written as 16-byte vectors start on 16-byte boundaries
static_assert(offsetof(Smem, red) % 16 == 0 && offsetof(Smem, rowinv) % 16 == 0 && offsetof(Smem, red2) % 16 == 0 &&
                  offsetof(Smem, ut) % 16 == 0 && offsetof(Smem, full) % 8 == 0 && offsetof(Smem, rc) % 16 == 0,
              "shared-memory layout");
static_assert(offsetof(Stage, q) % 16 == 0 && offsetof(Stage, k) % 16 == 0 && offsetof(Stage, v) % 16 == 0 &&
                  offsetof(Stage, g) % 16 == 0 && offsetof(Stage, r) % 16 == 0,
              "stage layout");
static_assert(offsetof(RowCoef, kl) % 16 == 0 && offsetof(RowCoef, h) % 16 == 0, "row data layout");

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

// Waits for the phase of parity `parity`; gives up (false) after limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long *bar, uint32_t parity,
                                                  unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > limit_ns) return false;
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

// named CTA barriers (ids 1-15; 0 is __syncthreads): arrive without waiting, or wait
__device__ __forceinline__ void bar_arrive(int id, int count)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// packed pair arithmetic (sm_100: one instruction for two fp32 lanes).  NV selects the
// compiler's float2 builtins (its own register pairing and scheduling) over inline PTX;
// which one the compiler turns into the faster code differs between the kernel's
// instantiations (measured), so each instantiation picks its own.
template <bool NV>
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    if constexpr (NV) return __ffma2_rn(a, b, c);
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

template <bool NV>
__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    if constexpr (NV) return __fadd2_rn(a, b);
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

template <bool NV>
__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    if constexpr (NV) return __fmul2_rn(a, b);
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

// (a & m) ^ c | (c & ~m) in one LOP3: keep a's bits under mask m, flip those
// set in c, and take c's bits elsewhere.
template <uint32_t M, uint32_t C>
__device__ __forceinline__ uint32_t masked_field(uint32_t a)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "n"(M), "n"(C));
    return d;
}

// ---------------------------------------------------------------- codecs
//
// unpack: the 8 codes of columns [8 cg, 8 cg + 8) of one packed row (in
// shared memory) as float pairs (first pass).  The b-bit two's complement code z becomes
// the offset code u = z + 2^(b-1) by flipping its top bit, u is placed in the
// mantissa of a power of two 2^E whose last mantissa bit weighs 1 (exact: 2^E + u)
// and 2^E + 2^(b-1) is subtracted (exact).  For 4 and 6 bits one LOP3 per code
// masks the field where it lies in the word, flips its top bit and sets the
// exponent: a field at bit offset f takes E = 23 - f, so no shifts are needed
// for fields that end below bit 23.
//
// store: the inverse, straight to the page in global memory, for requantised
// codes given as the bit patterns of fl(w inv + kMagicOut): 2^23 + u for 4
// and 6 bits, 1.5 * 2^23 + z for 8 bits.

template <int B> struct Codec;

template <> struct Codec<8> {
    static constexpr float kMagicOut = 12582912.0f;  // 1.5 * 2^23: low byte = z (two's complement)
    __device__ __forceinline__ static void store(uint8_t *rowg, int cg, const uint32_t b[8])
    {
        uint2 w;
        w.x = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
        w.y = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
        *reinterpret_cast<uint2 *>(rowg + cg * 8) = w;
    }
    template <bool NV>
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        const uint2 w = *reinterpret_cast<const uint2 *>(rowp + cg * 8);
        const uint32_t x0 = w.x ^ 0x80808080u, x1 = w.y ^ 0x80808080u;
        const float2 off = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
        z[0] = fadd2<NV>(make_float2(f_of(__byte_perm(x0, 0x4B000000u, 0x7650)), f_of(__byte_perm(x0, 0x4B000000u, 0x7651))), off);
        z[1] = fadd2<NV>(make_float2(f_of(__byte_perm(x0, 0x4B000000u, 0x7652)), f_of(__byte_perm(x0, 0x4B000000u, 0x7653))), off);
        z[2] = fadd2<NV>(make_float2(f_of(__byte_perm(x1, 0x4B000000u, 0x7650)), f_of(__byte_perm(x1, 0x4B000000u, 0x7651))), off);
        z[3] = fadd2<NV>(make_float2(f_of(__byte_perm(x1, 0x4B000000u, 0x7652)), f_of(__byte_perm(x1, 0x4B000000u, 0x7653))), off);
    }
};

template <> struct Codec<4> {
    static constexpr float kMagicOut = 8388616.0f;  // 2^23 + 8: mantissa = u = z + 8 in [1, 15]
    __device__ __forceinline__ static void store(uint8_t *rowg, int cg, const uint32_t b[8])
    {
        // b[t] = 0x4B000000 + u_t: sum_t b[t] 16^t = sum_t u_t 16^t + 0xFB000000 (mod 2^32)
        uint32_t acc = b[0];
#pragma unroll
        for (int t = 1; t < 8; ++t) acc += b[t] << (4 * t);
        *reinterpret_cast<uint32_t *>(rowg + cg * 4) = (acc - 0xFB000000u) ^ 0x88888888u;
    }
    template <bool NV>
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        // code t at bits [4t, 4t + 4); codes 5..7 are shifted down to offsets 0, 4, 8
        const uint32_t x = *reinterpret_cast<const uint32_t *>(rowp + cg * 4);
        const uint32_t t = x >> 20;
        const uint32_t c0 = masked_field<0xFu, 0x4B000008u>(x);       // 2^23 + u
        const uint32_t c1 = masked_field<0xF0u, 0x49000080u>(x);      // 2^19 + u
        const uint32_t c2 = masked_field<0xF00u, 0x47000800u>(x);     // 2^15 + u
        const uint32_t c3 = masked_field<0xF000u, 0x45008000u>(x);    // 2^11 + u
        const uint32_t c4 = masked_field<0xF0000u, 0x43080000u>(x);   // 2^7 + u
        const uint32_t c5 = masked_field<0xFu, 0x4B000008u>(t);
        const uint32_t c6 = masked_field<0xF0u, 0x49000080u>(t);
        const uint32_t c7 = masked_field<0xF00u, 0x47000800u>(t);
        z[0] = fadd2<NV>(make_float2(f_of(c0), f_of(c1)), make_float2(-8388616.0f, -524296.0f));
        z[1] = fadd2<NV>(make_float2(f_of(c2), f_of(c3)), make_float2(-32776.0f, -2056.0f));
        z[2] = fadd2<NV>(make_float2(f_of(c4), f_of(c5)), make_float2(-136.0f, -8388616.0f));
        z[3] = fadd2<NV>(make_float2(f_of(c6), f_of(c7)), make_float2(-524296.0f, -32776.0f));
    }
};

template <> struct Codec<6> {
    // A row is 16 groups of 8 codes; group cg is a 48-bit string (code p at bits
    // [6p, 6p + 6)) kept as a 32-bit word at byte 4 cg and a 16-bit half at byte
    // 64 + 2 cg, so both accesses are aligned and no thread straddles another's.
    static constexpr float kMagicOut = 8388640.0f;  // 2^23 + 32: mantissa = u = z + 32 in [1, 63]
    __device__ __forceinline__ static void store(uint8_t *rowg, int cg, const uint32_t b[8])
    {
        // b[t] = 0x4B000000 + u_t; the 0x4B000000 parts cancel or shift out except a constant
        uint32_t lo = b[0] + (b[1] << 6) + (b[2] << 12) + (b[3] << 18) + (b[4] << 24) + (b[5] << 30);
        lo = (lo - 0x0B000000u) ^ 0x20820820u;
        const uint32_t hi = ((b[5] >> 2) + (b[6] << 4) + (b[7] << 10)) ^ 0x8208u;
        *reinterpret_cast<uint32_t *>(rowg + cg * 4) = lo;
        *reinterpret_cast<uint16_t *>(rowg + 64 + cg * 2) = static_cast<uint16_t>(hi);
    }
    template <bool NV>
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        const uint32_t lo = *reinterpret_cast<const uint32_t *>(rowp + cg * 4);
        const uint32_t hi = *reinterpret_cast<const uint16_t *>(rowp + 64 + cg * 2);
        const uint32_t x = lo >> 18;                     // codes 3, 4 at offsets 0, 6
        const uint32_t y = __funnelshift_r(lo, hi, 30);  // codes 5, 6, 7 at offsets 0, 6, 12
        const uint32_t c0 = masked_field<0x3Fu, 0x4B000020u>(lo);     // 2^23 + u
        const uint32_t c1 = masked_field<0xFC0u, 0x48000800u>(lo);    // 2^17 + u
        const uint32_t c2 = masked_field<0x3F000u, 0x45020000u>(lo);  // 2^11 + u
        const uint32_t c3 = masked_field<0x3Fu, 0x4B000020u>(x);
        const uint32_t c4 = masked_field<0xFC0u, 0x48000800u>(x);
        const uint32_t c5 = masked_field<0x3Fu, 0x4B000020u>(y);
        const uint32_t c6 = masked_field<0xFC0u, 0x48000800u>(y);
        const uint32_t c7 = masked_field<0x3F000u, 0x45020000u>(y);
        z[0] = fadd2<NV>(make_float2(f_of(c0), f_of(c1)), make_float2(-8388640.0f, -131104.0f));
        z[1] = fadd2<NV>(make_float2(f_of(c2), f_of(c3)), make_float2(-2080.0f, -8388640.0f));
        z[2] = fadd2<NV>(make_float2(f_of(c4), f_of(c5)), make_float2(-131104.0f, -8388640.0f));
        z[3] = fadd2<NV>(make_float2(f_of(c6), f_of(c7)), make_float2(-131104.0f, -2080.0f));
    }
};

// FP16 pivot rows ("method steps", step 1: pivot units are read in FP16
// directly): the row holds mu = X / (r c) as 128 binary16 values; a thread's 8
// columns are one 16-byte vector.  The scale slot of the row holds 1, so the
// row enters both passes like a quantized row whose codes are mu.
struct Pivot16 {
    template <bool NV>
    __device__ __forceinline__ static void unpack(const uint8_t *rowp, int cg, float2 z[4])
    {
        const uint4 w = *reinterpret_cast<const uint4 *>(rowp + cg * 16);
        z[0] = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
        z[1] = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
        z[2] = __half22float2(*reinterpret_cast<const __half2 *>(&w.z));
        z[3] = __half22float2(*reinterpret_cast<const __half2 *>(&w.w));
    }
    // t: the new mu of the 8 columns, rounded once to binary16 (nearest even)
    __device__ __forceinline__ static void store(uint8_t *rowg, int cg, const float2 t[4])
    {
        __half2 h[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) h[p] = __float22half2_rn(t[p]);
        uint4 w;
        w.x = *reinterpret_cast<const uint32_t *>(&h[0]);
        w.y = *reinterpret_cast<const uint32_t *>(&h[1]);
        w.z = *reinterpret_cast<const uint32_t *>(&h[2]);
        w.w = *reinterpret_cast<const uint32_t *>(&h[3]);
        *reinterpret_cast<uint4 *>(rowg + cg * 16) = w;
    }
};

template <bool NV>
__device__ __forceinline__ void unpack_any(int b, const uint8_t *rowp, int cg, float2 z[4])
{
    if (b == 16) Pivot16::unpack<NV>(rowp, cg, z);
    else if (b == 8) Codec<8>::unpack<NV>(rowp, cg, z);
    else if (b == 6) Codec<6>::unpack<NV>(rowp, cg, z);
    else Codec<4>::unpack<NV>(rowp, cg, z);
}

__device__ __forceinline__ void store_any(int b, uint8_t *rowg, int cg, const uint32_t bits[8])
{
    if (b == 8) Codec<8>::store(rowg, cg, bits);
    else if (b == 6) Codec<6>::store(rowg, cg, bits);
    else Codec<4>::store(rowg, cg, bits);
}

__device__ __forceinline__ float magic_out(int b)
{
    return b == 8 ? Codec<8>::kMagicOut : (b == 6 ? Codec<6>::kMagicOut : Codec<4>::kMagicOut);
}


// ---------------------------------------------------------------- one tile
//
// Thread (rg, cg) = (2 warp + lane / 16, lane % 16) owns rows [8 rg, 8 rg + 8)
// and columns [8 cg, 8 cg + 8); z[ii][p] holds columns 8 cg + 2 p, + 1 of row
// 8 rg + ii in registers across both passes: first the old codes, then the
// updated row values w.
//
// Pass 1: unpack the old codes, accumulate the two column sums and leave
// per-warp partials in red.  B = 4, 6, 8: every row has B bits, at
// 16 B i (GDN) or, with PR, at the row table's offsets (a KDA warp whose
// rows share one width); B = 0: per-row widths (KDA).
template <int B, int SB, bool FIT, bool NV, bool ACC = true, bool PR = false>
__device__ __forceinline__ void pass1(Smem &sm, const Stage &S, const RowCoef &R, float2 z[8][4])
{
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int rgl = lane >> 4, cg = lane & 15;
    const int i0 = (warp * 2 + rgl) * 8;
    float2 av[4], ay[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) av[p] = ay[p] = make_float2(0.0f, 0.0f);
    // a fitted page's pivot rows hold X / r: their values enter as mu / c_j, like codes
    float2 ic[4];
    if (B == 0 && FIT) {
        const float4 a = *reinterpret_cast<const float4 *>(S.page + SB * kD + 32 * cg);
        const float4 b = *reinterpret_cast<const float4 *>(S.page + SB * kD + 32 * cg + 16);
        ic[0] = make_float2(rcp_approx(a.x), rcp_approx(a.y));
        ic[1] = make_float2(rcp_approx(a.z), rcp_approx(a.w));
        ic[2] = make_float2(rcp_approx(b.x), rcp_approx(b.y));
        ic[3] = make_float2(rcp_approx(b.z), rcp_approx(b.w));
    }
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        if (B != 0 && PR) Codec<B == 0 ? 8 : B>::template unpack<NV>(S.page + R.off[i], cg, z[ii]);
        else if (B != 0) Codec<B == 0 ? 8 : B>::template unpack<NV>(S.page + SB * kD + (FIT ? kFitBytes : 0) + 16 * B * i, cg, z[ii]);
        else unpack_any<NV>(R.bits[i], S.page + R.off[i], cg, z[ii]);
        if (B == 0 && FIT && R.bits[i] == 16) {
#pragma unroll
            for (int p = 0; p < 4; ++p) z[ii][p] = fmul2<NV>(z[ii][p], ic[p]);
        }
        if constexpr (ACC) {
            const float4 kl = R.kl[i];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                av[p] = ffma2<NV>(make_float2(kl.x, kl.y), z[ii][p], av[p]);
                ay[p] = ffma2<NV>(make_float2(kl.z, kl.w), z[ii][p], ay[p]);
            }
        }
    }
    if constexpr (ACC) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            av[p] = fadd2<NV>(av[p], make_float2(__shfl_xor_sync(0xffffffffu, av[p].x, 16),
                                             __shfl_xor_sync(0xffffffffu, av[p].y, 16)));
            ay[p] = fadd2<NV>(ay[p], make_float2(__shfl_xor_sync(0xffffffffu, ay[p].x, 16),
                                             __shfl_xor_sync(0xffffffffu, ay[p].y, 16)));
        }
        // half 0 keeps the v-sums, half 1 the y-sums; column j of a sum sits at
        // ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3) (conflict-free 16-byte stores)
        const float2 *src = rgl == 0 ? av : ay;
        float *dst = &sm.red[warp * kRedStride + rgl * 128 + cg * 4];
        *reinterpret_cast<float4 *>(dst) = make_float4(src[0].x, src[0].y, src[1].x, src[1].y);
        *reinterpret_cast<float4 *>(dst + 64) = make_float4(src[2].x, src[2].y, src[3].x, src[3].y);
    }
}

// Column handled by epilogue thread t (0..127): column t, so that a warp's y
// stores are one contiguous 128-byte line (whole lines also when y is page-locked
// host memory written across the bus); its reads of the partial sums meet 2-way
// bank conflicts, which measured cheaper than scattered y stores.
__device__ __forceinline__ int epilogue_column(int t) { return t; }

// Per column (threads 0..127), one tile after pass 2 wrote its partial sums:
// the refitted factor c_j <- c_j sum_i A_i z'_ij w_ij / sum_i B_i z'_ij^2
// (= sum_i w_i^2 v_ij X_ij / sum_i w_i^2 v_ij^2 with v_ij = s'_i r_i z'_ij and
// X_ij = c_j e~_i w_ij), stored into that tile's page; a column whose codes
// are all zero keeps its factor.
template <int SB>
__device__ __forceinline__ void fit_finish(Smem &sm, int parity)
{
    if (!sm.fit_pending[parity]) return;
    const int j = epilogue_column(threadIdx.x);
    const int at = ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3);
    float num = 0.0f, den = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        num += sm.red2[w * 256 + at];
        den += sm.red2[w * 256 + 128 + at];
    }
    const float c_old = sm.fitc[j];
    const float c_new = den > 0.0f ? c_old * __fdiv_rn(num, den) : c_old;
    if (!isfinite(c_new)) atomicOr(&sm.flags, kErrNonFinite);
    reinterpret_cast<float *>(sm.fit_page[parity] + SB * kD)[j] = c_new;
}

// Per column (threads 0..127): v_old, u, y, u / c.  The write-back takes
// u / c from the readout's buffer (prefetched into the stage's v) instead.
template <int MODE, int SB, bool FIT>
__device__ __forceinline__ void column_epilogue(Smem &sm, const Stage &S, const RowCoef &R,
                                                const DecodeIO &io, int tile, float beta)
{
    const int j = epilogue_column(threadIdx.x);
    // the column factors this tile's codes are read and taken with
    const float cj = FIT ? reinterpret_cast<const float *>(S.page + SB * kD)[j] : S.c[j];
    if (FIT && MODE != kReadout) sm.fitc[j] = cj;
    // column j's slot in the partial sums, and in ut (columns 8 g .. 8 g + 3 of a column group
    // g at 4 g, columns 8 g + 4 .. 8 g + 7 at 64 + 4 g: pass 2 reads them as 16-byte vectors)
    const int at = ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3);
    if (MODE == kWriteback) {
        sm.ut[at] = S.v[j];
        return;
    }
    float vz = 0.0f, yz = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        vz += sm.red[w * kRedStride + at];
        yz += sm.red[w * kRedStride + 128 + at];
    }
    const float u = beta * (S.v[j] - cj * vz);
    const float kq = (R.kqp[0] + R.kqp[1]) + (R.kqp[2] + R.kqp[3]);
    const float yj = fmaf(u, kq, cj * yz);
    io.y[static_cast<size_t>(tile) * kD + j] = yj;
    const float ut = u * rcp_approx(cj);
    if (MODE == kReadout) io.u_out[static_cast<size_t>(tile) * kD + j] = ut;
    else sm.ut[at] = ut;
    if (!isfinite(u) || !isfinite(yj)) atomicOr(&sm.flags, kErrNonFinite);
}

// Per position (threads 128..255) of the next tile: decayed scale e_i of its
// row i and the coefficients both passes need; warps 4-7 also form k.q.
template <int KIND, int SB, int MODE, bool FIT>
__device__ __forceinline__ void row_setup(Smem &sm, const Stage &S, RowCoef &R, int s)
{
    const int pos = threadIdx.x - kD;
    const bool valid = sm.stage_valid[s] != 0;
    if (pos == 0) {
        R.page = sm.stage_page[s];
        R.valid = valid;
    }
    if (!valid) return;
    const int r = KIND == STQ_KDA ? S.perm[pos] : pos;
    const float sc = SB == 4 ? reinterpret_cast<const float *>(S.page)[r]
                             : __half2float(reinterpret_cast<const __half *>(S.page)[r]);
    const float g = KIND == STQ_GDN ? sm.alpha[s] : S.g[r];
    const float rr = S.r[r];
    const float e = (g * sc) * rr;
    const float kr = S.k[r];
    const float qr = MODE == kWriteback ? 0.0f : S.q[r];  // the write-back loads no q
    const float ka = kr * e, la = qr * e;
    const float hq = kr * rcp_approx(e);
    const bool dropped = !(e != 0.0f && fabsf(hq) <= 1e30f);
    R.kl[pos] = make_float4(ka, ka, la, la);
    R.h[pos] = dropped ? kr : hq;
    R.mrq[pos] = (dropped ? 1.0f : e) * S.inv_rq[r];
    if (FIT) {
        const float wr = sm.stage_w[s][r] * rr;
        R.fb[pos] = wr * wr;
    }
    R.off[pos] = S.row_off[r];
    R.bits[pos] = S.row_bits[r];
    if (KIND == STQ_KDA) {
        R.row[pos] = static_cast<uint8_t>(r);
        // pass warp pos / 16 takes positions [16 (pos / 16), + 16): one width for all, or 0
        const uint32_t same = __match_any_sync(0xffffffffu, static_cast<uint32_t>(S.row_bits[r]));
        const uint32_t half = 0xFFFFu << (pos & 16);
        if ((pos & 15) == 0) R.wbits[pos >> 4] = (same & half) == half ? S.row_bits[r] : 0;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, dropped);
    if ((pos & 31) == 0) R.deg[pos >> 5] = bal;
    if (!isfinite(e)) atomicOr(&sm.flags, kErrNonFinite);
    float a = kr * qr;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if ((pos & 31) == 0) R.kqp[pos >> 5] = a;
}

// Pass 2: w = z + h u~, row absmax (8 columns per thread, then the 16 column
// groups of the half-warp through shared memory), new scale, requantise,
// store codes and scales to the page in global memory.
template <int B, int SB, bool FIT, bool NV, bool PR = false>
__device__ __forceinline__ void pass2(Smem &sm, const RowCoef &R, const Stage &S, float2 z[8][4])
{
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int rgl = lane >> 4, cg = lane & 15;
    const int i0 = (warp * 2 + rgl) * 8;
    float2 ut2[4];
    {
        const float4 a = *reinterpret_cast<const float4 *>(&sm.ut[cg * 4]);
        const float4 b = *reinterpret_cast<const float4 *>(&sm.ut[64 + cg * 4]);
        ut2[0] = make_float2(a.x, a.y);
        ut2[1] = make_float2(a.z, a.w);
        ut2[2] = make_float2(b.x, b.y);
        ut2[3] = make_float2(b.z, b.w);
    }
    const uint32_t deg = (R.deg[i0 >> 5] >> (i0 & 31)) & 0xFFu;
    float hs[8];
    {
        const float4 ha = *reinterpret_cast<const float4 *>(&R.h[i0]);
        const float4 hb = *reinterpret_cast<const float4 *>(&R.h[i0 + 4]);
        hs[0] = ha.x; hs[1] = ha.y; hs[2] = ha.z; hs[3] = ha.w;
        hs[4] = hb.x; hs[5] = hb.y; hs[6] = hb.z; hs[7] = hb.w;
    }
    if (deg == 0) {
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) {
            const float2 h2 = make_float2(hs[ii], hs[ii]);
#pragma unroll
            for (int p = 0; p < 4; ++p) z[ii][p] = ffma2<NV>(h2, ut2[p], z[ii][p]);
        }
    } else {
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) {
            const float2 h2 = make_float2(hs[ii], hs[ii]);
            if (!((deg >> ii) & 1u)) {
#pragma unroll
                for (int p = 0; p < 4; ++p) z[ii][p] = ffma2<NV>(h2, ut2[p], z[ii][p]);
            } else {
#pragma unroll
                for (int p = 0; p < 4; ++p) z[ii][p] = fmul2<NV>(h2, ut2[p]);
            }
        }
    }
    float mx[8];
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        float m = max3(fabsf(z[ii][0].x), fabsf(z[ii][0].y), fabsf(z[ii][1].x));
        m = max3(m, fabsf(z[ii][1].y), fabsf(z[ii][2].x));
        m = max3(m, fabsf(z[ii][2].y), fabsf(z[ii][3].x));
        mx[ii] = fmaxf(m, fabsf(z[ii][3].y));
    }
    // row maxima: this thread's 8 partials -> shared; lane (rgl, cg) then reduces row
    // 8 rg + (cg & 7) over the 8 column groups of half cg >> 3.  Column group m of a half
    // sits 36 floats from group m - 1, so that both the 16-byte stores (each quarter
    // warp on distinct banks) and the scalar loads are free of bank conflicts.
    float *rm = &sm.red[warp * kRedStride];
    {
        float4 *dst = reinterpret_cast<float4 *>(&rm[(cg & 7) * 36 + rgl * 16 + (cg >> 3) * 8]);
        dst[0] = make_float4(mx[0], mx[1], mx[2], mx[3]);
        dst[1] = make_float4(mx[4], mx[5], mx[6], mx[7]);
    }
    __syncwarp();
    uint8_t *page = R.page;
    bool clip = false;  // binary16 scale below a / q_b in the subnormal range: codes need clipping
    {
        const int ii = cg & 7, half = cg >> 3;
        const float *src = &rm[rgl * 16 + half * 8 + ii];
        float m = max3(src[0], src[36], src[72]);
        m = max3(m, src[108], src[144]);
        m = max3(m, src[180], src[216]);
        m = fmaxf(m, src[252]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        if (half == 0) {
            const int i = i0 + ii;                 // position
            const int row = B != 0 && !PR ? i : R.row[i];  // its row: the scale slot
            const int b = B != 0 ? B : R.bits[i];
            const float qb = static_cast<float>((1 << (b - 1)) - 1);
            const float mrq = R.mrq[i];
            float inv = 0.0f, snew = 0.0f;
            if (B == 0 && b == 16) {
                // pivot row: the scale slot keeps 1; mu beyond the binary16 range is reported
                if (!(fabsf(mrq) * m < 65520.0f)) atomicOr(&sm.flags, kErrNonFinite);
                if (SB == 4) reinterpret_cast<float *>(page)[row] = 1.0f;
                else reinterpret_cast<__half *>(page)[row] = __float2half_rn(1.0f);
            } else if (SB == 4) {
                if (m >= 1e-30f && m <= 3.0e38f) {
                    inv = copysignf(qb * rcp_approx(m), mrq);
                    snew = fabsf(mrq) * m;
                } else if (m > 0.0f && m < 1e-30f) {
                    inv = copysignf(__fdiv_rn(qb, m), mrq);
                    snew = fabsf(mrq) * m;
                } else if (!(m == 0.0f)) {
                    atomicOr(&sm.flags, kErrNonFinite);
                }
                reinterpret_cast<float *>(page)[row] = snew;
                if (FIT) {
                    // A = w^2 r e~ s' = (w r)^2 q_b mrq s', since mrq = e~ / (r q_b)
                    sm.rowA[i] = ((R.fb[i] * qb) * mrq) * snew;
                    sm.rowB[i] = (R.fb[i] * snew) * snew;
                }
            } else {
                // binary16 scale: s16 = half(a / q_b); the codes are rounded from
                // mu / s16 = w (e / r) / s16 = w mrq q_b / s16
                const float s = fabsf(mrq) * m;
                const __half s16 = __float2half_rn(s);
                const float sf = __half2float(s16);
                if (sf > 0.0f && sf <= 65504.0f) inv = mrq * qb * rcp_approx(sf);
                else if (!(sf == 0.0f)) atomicOr(&sm.flags, kErrNonFinite);  // overflow or NaN
                // for a normal binary16 scale s / s16 <= 1 + 2^-11, so |w inv| <= q_b (1 + 2^-11)
                // rounds to at most q_b (q_b <= 127); only a subnormal s16 can round further down
                clip = sf < s && sf < 6.103515625e-05f;
                reinterpret_cast<__half *>(page)[row] = s16;
                if (FIT) {
                    const float sv = sf <= 65504.0f ? sf : 0.0f;
                    sm.rowA[i] = ((R.fb[i] * qb) * mrq) * sv;
                    sm.rowB[i] = (R.fb[i] * sv) * sv;
                }
            }
            sm.rowinv[i] = inv;
        }
    }
    // bit ii: row i0 + ii needs its codes clipped (lanes 0-7 and 16-23 decided rows of
    // row groups 2 warp and 2 warp + 1)
    const uint32_t clipm = SB == 2 ? (__ballot_sync(0xffffffffu, clip) >> (rgl * 16)) & 0xFFu : 0u;
    __syncwarp();
    const float4 ia = *reinterpret_cast<const float4 *>(&sm.rowinv[i0]);
    const float4 ib = *reinterpret_cast<const float4 *>(&sm.rowinv[i0 + 4]);
    const float invs[8] = {ia.x, ia.y, ia.z, ia.w, ib.x, ib.y, ib.z, ib.w};
    // column fit: per-column sums of A_i z'_ij w_ij and B_i z'_ij^2 over this thread's rows
    float2 fnum[4], fden[4];
    if (FIT) {
#pragma unroll
        for (int p = 0; p < 4; ++p) fnum[p] = fden[p] = make_float2(0.0f, 0.0f);
    }
    uint8_t *rows = page + SB * kD + (FIT ? kFitBytes : 0);
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
        const int i = i0 + ii;
        const int b = B != 0 ? B : R.bits[i];
        if (B == 0 && b == 16) {
            // pivot row: mu = X / (r c) = (e / r) w, with R.mrq = e / r for a pivot row; a
            // fitted page's pivot row keeps mu = X / r = c_j (e / r) w (c_j: the factors
            // this tile's codes were taken with, still in the stage)
            const float2 m2 = make_float2(R.mrq[i], R.mrq[i]);
            float2 t[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) t[p] = fmul2<NV>(z[ii][p], m2);
            if (FIT) {
                const float4 a = *reinterpret_cast<const float4 *>(S.page + SB * kD + 32 * cg);
                const float4 b = *reinterpret_cast<const float4 *>(S.page + SB * kD + 32 * cg + 16);
                t[0] = fmul2<NV>(t[0], make_float2(a.x, a.y));
                t[1] = fmul2<NV>(t[1], make_float2(a.z, a.w));
                t[2] = fmul2<NV>(t[2], make_float2(b.x, b.y));
                t[3] = fmul2<NV>(t[3], make_float2(b.z, b.w));
            }
            Pivot16::store(page + R.off[i], cg, t);
            continue;
        }
        const float mg = B != 0 ? Codec<B == 0 ? 8 : B>::kMagicOut : magic_out(b);
        const float2 inv2 = make_float2(invs[ii], invs[ii]), mg2 = make_float2(mg, mg);
        uint32_t bits[8];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            float2 t = ffma2<NV>(z[ii][p], inv2, mg2);
            if (SB == 2 && ((clipm >> ii) & 1u)) {
                // the binary16 scale rounded below a / q_b by up to half a subnormal step:
                // clip the rounded quotient to [-q_b, q_b]
                const float qb = static_cast<float>((1 << (b - 1)) - 1);
                t.x = fminf(fmaxf(t.x, mg - qb), mg + qb);
                t.y = fminf(fmaxf(t.y, mg - qb), mg + qb);
            }
            bits[2 * p] = __float_as_uint(t.x);
            bits[2 * p + 1] = __float_as_uint(t.y);
            if (FIT) {
                // z' = t - mg exactly (the new code); A z' w and B z'^2 into the column sums
                const float2 zq = fadd2<NV>(t, make_float2(-mg, -mg));
                const float A = sm.rowA[i], Bc = sm.rowB[i];
                fnum[p] = ffma2<NV>(make_float2(A, A), fmul2<NV>(zq, z[ii][p]), fnum[p]);
                fden[p] = ffma2<NV>(make_float2(Bc, Bc), fmul2<NV>(zq, zq), fden[p]);
            }
        }
        if (B != 0 && PR) Codec<B == 0 ? 8 : B>::store(page + R.off[i], cg, bits);
        else if (B != 0) Codec<B == 0 ? 8 : B>::store(rows + 16 * B * i, cg, bits);
        else store_any(b, page + R.off[i], cg, bits);
    }
    if (FIT) {
        // per-warp partials, laid out as pass 1's column sums (half 0 numerators, half 1 denominators)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            fnum[p] = fadd2<NV>(fnum[p], make_float2(__shfl_xor_sync(0xffffffffu, fnum[p].x, 16),
                                                 __shfl_xor_sync(0xffffffffu, fnum[p].y, 16)));
            fden[p] = fadd2<NV>(fden[p], make_float2(__shfl_xor_sync(0xffffffffu, fden[p].x, 16),
                                                 __shfl_xor_sync(0xffffffffu, fden[p].y, 16)));
        }
        const float2 *src = rgl == 0 ? fnum : fden;
        float *dst = &sm.red2[warp * 256 + rgl * 128 + cg * 4];
        *reinterpret_cast<float4 *>(dst) = make_float4(src[0].x, src[0].y, src[1].x, src[1].y);
        *reinterpret_cast<float4 *>(dst + 64) = make_float4(src[2].x, src[2].y, src[3].x, src[3].y);
    }
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
__device__ __forceinline__ void issue(Smem &sm, int s, const PoolView &p, const TileRef &t, uint32_t stall_tx = 0)
{
    Stage &S = sm.st[s];
    sm.stage_page[s] = t.page;
    sm.stage_w[s] = p.t.w + static_cast<size_t>(t.h) * kD;
    // a page larger than a stage is a GDN FP16 pivot head, advanced by its own kernel
    const bool mine = t.valid && t.bytes <= static_cast<uint32_t>(kMaxPage);
    sm.stage_valid[s] = mine;
    if (!mine) {
        if (!t.valid) atomicOr(&sm.flags, kErrIndex);
        mbar_arrive(&sm.full[s]);  // completes the phase with no data; the tile is skipped
        return;
    }
    // stall_tx (a test hook, 0 otherwise): bytes that no copy delivers, so that the wait runs out
    mbar_arrive_expect_tx(&sm.full[s], t.bytes + kHeadBlock + stall_tx);
    bulk_load(S.page, t.page, t.bytes, &sm.full[s]);
    bulk_load(S.r, p.t.block + static_cast<size_t>(t.h) * kHeadBlock, kHeadBlock, &sm.full[s]);
}

// Asynchronous prefetch, one cp.async group per thread per tile (issued after
// the first barrier of tile i, waited with wait_group 1 before the first
// barrier of tile i + 2): q, k, v (and the KDA decay), beta, alpha of tile
// i + 3 into its stage, and the raw location {req, slot, head offset, page
// bytes} of tile i + 5 = (request entry n5, head h5).  The small copies are
// spread over warps 5-7, which have the least other work at this point.
// cp.async of tile `tile`'s q, k, v (and the KDA decay), beta and alpha into stage s
// (warps 0-3 the vectors, threads 160 and 192 the scalars); the caller commits.
template <int KIND, int MODE>
__device__ __forceinline__ void prefetch_vectors(Smem &sm, const DecodeIO &io, int s, int tile)
{
    const int t = threadIdx.x;
    Stage &S = sm.st[s];
    const size_t base = static_cast<size_t>(tile) * kD + 4 * (t & 31);
    if (t < 32) {
        if (MODE != kWriteback) cp_async16(&S.q[4 * t], io.q + base);
    }
    else if (t < 64) cp_async16(&S.k[4 * (t - 32)], io.k + base);
    else if (t < 96) cp_async16(&S.v[4 * (t - 64)], io.v + base);
    else if (t < 128) {
        if (KIND == STQ_KDA) cp_async16(&S.g[4 * (t - 96)], io.gate + base);
    } else if (t == 160) {
        if (MODE != kWriteback) cp_async4(&sm.beta[s], io.beta + tile);
    } else if (t == 192) {
        if (KIND == STQ_GDN) cp_async4(&sm.alpha[s], io.gate + tile);
    }
}

template <int KIND, int MODE>
__device__ __forceinline__ void prefetch(Smem &sm, const PoolView &p, const DecodeIO &io, int i, int t3, int t5,
                                         int n5, int h5, int tiles)
{
    const int t = threadIdx.x;
    if (t3 < tiles) prefetch_vectors<KIND, MODE>(sm, io, (i + 3) % kStages, t3);
    if (t5 < tiles && t >= 224 && t < 228) {
        uint32_t *dst = &sm.raw[(i + 5) & 7][t - 224];
        const void *src = t == 224 ? static_cast<const void *>(io.req_idx + n5)
                        : t == 225 ? static_cast<const void *>(io.slot_idx + n5)
                        : t == 226 ? static_cast<const void *>(p.t.head_off + h5)
                                   : static_cast<const void *>(p.t.page_bytes + h5);
        cp_async4(dst, src);
        if (t == 224) dst[4] = static_cast<uint32_t>(h5);
    }
    cp_async_commit();
}

__device__ __forceinline__ TileRaw raw_from_smem(const Smem &sm, int k)
{
    TileRaw r;
    r.h = static_cast<int>(sm.raw[k & 7][4]);
    r.req = static_cast<int>(sm.raw[k & 7][0]);
    r.slot = static_cast<int>(sm.raw[k & 7][1]);
    r.hoff = sm.raw[k & 7][2];
    r.bytes = sm.raw[k & 7][3];
    return r;
}

// Persistent CTA: tiles first, first + G, first + 2G, ... (G = gridDim.x).
// Per tile i (stage i % 4, row data rc[i % 2]):
//   all:       pass 1 of tile i                                        | __syncthreads
//   thread 96: issue tile i + 3 (page and head block) into the stage of tile i - 1
//   all:       cp.async prefetch of tile i + 3's vectors, tile i + 5's location
//   warps 0-3: column epilogue of tile i (y, u / c)   | arrive 1, sync 2 (warps 0-3)
//   warps 4-7: wait for tile i + 1's stage, its row coefficients   | arrive 3, sync 1
//   all:       pass 2 of tile i (codes held in registers; new codes and scales to global memory)
//   warps 0-3: sync 3 (tile i + 1's row data is in) before their next pass 1
// Named barriers let warps 0-3 start pass 2 as soon as the four epilogue warps
// are done, without waiting for warps 4-7's row setup of the next tile.  A
// stage is last read before barrier 1 of its tile (pass 2 reads only registers,
// the row data and, for fitted pivot rows, the column factors before the next
// __syncthreads); thread 96 refills it after the first barrier of the next tile.
template <int KIND, int SB, int MODE, bool FIT>
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
        sm.stop = 0;
        sm.fit_pending[0] = sm.fit_pending[1] = 0;
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    // prologue: the locations of the first five tiles (thread a loads tile a's) and,
    // asynchronously, the vectors of the first three, all in flight together
    if (tid < 5 && first + tid * G < tiles) {
        const TileRaw r = load_raw(p, io, first + tid * G);
        sm.raw[tid][0] = static_cast<uint32_t>(r.req);
        sm.raw[tid][1] = static_cast<uint32_t>(r.slot);
        sm.raw[tid][2] = r.hoff;
        sm.raw[tid][3] = r.bytes;
        sm.raw[tid][4] = static_cast<uint32_t>(r.h);
    }
    for (int a = 0; a < 3; ++a)
        if (first + a * G < tiles) prefetch_vectors<KIND, MODE>(sm, io, a, first + a * G);
    cp_async_commit();
    __syncthreads();  // barriers initialised, locations in
    if (tid == 0)
        for (int a = 0; a < 3; ++a)
            if (first + a * G < tiles)
                issue<KIND>(sm, a, p, resolve(p, raw_from_smem(sm, a)), first == 0 && a == 0 ? p.stall_tx : 0u);
    cp_async_wait<0>();
    __syncthreads();  // the first vectors and the stages' validity are visible
    bool timed_out = false;
    if (tid >= kD) {
        // warp-uniform outcome: row_setup's shuffles need every lane
        if (__all_sync(0xffffffffu, mbar_wait_bounded(&sm.full[0], 0, p.wait_ns))) row_setup<KIND, SB, MODE, FIT>(sm, sm.st[0], sm.rc[0], 0);
        else timed_out = true;
    }
    timed_out = __syncthreads_or(timed_out) != 0;

    // (request entry, head) of tile first + 5 G, advanced by G per tile without a division
    const int gq = G / p.H, gr = G - gq * p.H;
    int n5 = (first + 5 * G) / p.H;
    int h5 = first + 5 * G - n5 * p.H;
    int i = 0;
    for (int tile = first; tile < tiles && !timed_out; tile += G, ++i) {
        const int s = i % kStages;
        const RowCoef &R = sm.rc[i & 1];
        const Stage &S = sm.st[s];
        const bool valid = R.valid != 0;
        const int b = valid ? R.bits[0] : 8;
        float2 z[8][4];
        constexpr bool kAcc = MODE != kWriteback;
        constexpr bool kNV = KIND == STQ_GDN && !FIT;  // the builtins measure faster only here
        if (valid) {
            if constexpr (KIND == STQ_KDA) {
                // the one width of this warp's rows, or the per-row path (per-row widths and
                // pivot rows; the whole pool takes it when any of its tiles needs it)
                const int wb = p.per_row ? 0 : R.wbits[tid >> 5];
                if (wb == 6) pass1<6, SB, FIT, kNV, kAcc, true>(sm, S, R, z);
                else if (wb == 8) pass1<8, SB, FIT, kNV, kAcc, true>(sm, S, R, z);
                else if (wb == 4) pass1<4, SB, FIT, kNV, kAcc, true>(sm, S, R, z);
                else pass1<0, SB, FIT, kNV, kAcc>(sm, S, R, z);
            }
            else if (b == 8) pass1<8, SB, FIT, kNV, kAcc>(sm, S, R, z);
            else if (b == 6) pass1<6, SB, FIT, kNV, kAcc>(sm, S, R, z);
            else pass1<4, SB, FIT, kNV, kAcc>(sm, S, R, z);
        }
        cp_async_wait<1>();
        __syncthreads();
        if (tid == 96 && tile + 3 * G < tiles)  // warp 3: no vector prefetch for GDN
            issue<KIND>(sm, (i + 3) % kStages, p, resolve(p, raw_from_smem(sm, i + 3)));
        prefetch<KIND, MODE>(sm, p, io, i, tile + 3 * G, tile + 5 * G, n5, h5, tiles);
        n5 += gq;
        h5 += gr;
        if (h5 >= p.H) {
            h5 -= p.H;
            ++n5;
        }
        // barrier 1: u~ of this tile ready (warps 0-3 arrive, warps 4-7 wait); barrier 2: among
        // warps 0-3, every epilogue read of the partial sums done; barrier 3: the next tile's
        // row data ready (warps 4-7 arrive, warps 0-3 wait before their next pass 1)
        if (tid < kD) {
            constexpr bool kFits = FIT && MODE != kReadout;
            if (kFits) fit_finish<SB>(sm, (i + 1) & 1);  // the previous tile's factors
            if (valid) column_epilogue<MODE, SB, FIT>(sm, S, R, io, tile, sm.beta[s]);
            if (kFits && tid == 0) {
                sm.fit_page[i & 1] = R.page;
                sm.fit_pending[i & 1] = valid;
            }
            bar_arrive(1, kThreads);
            bar_sync(2, kD);
        } else {
            if (tile + G < tiles) {
                const int sn = (i + 1) % kStages;
                if (__all_sync(0xffffffffu, mbar_wait_bounded(&sm.full[sn], ((i + 1) / kStages) & 1, p.wait_ns)))
                    row_setup<KIND, SB, MODE, FIT>(sm, sm.st[sn], sm.rc[(i + 1) & 1], sn);
                else if ((tid & 31) == 0)
                    sm.stop = 1;
            }
            bar_arrive(3, kThreads);
            bar_sync(1, kThreads);
            timed_out = sm.stop != 0;
        }
        if (valid && MODE != kReadout) {
            if constexpr (KIND == STQ_KDA) {
                const int wb = p.per_row ? 0 : R.wbits[tid >> 5];
                if (wb == 6) pass2<6, SB, FIT, kNV, true>(sm, R, S, z);
                else if (wb == 8) pass2<8, SB, FIT, kNV, true>(sm, R, S, z);
                else if (wb == 4) pass2<4, SB, FIT, kNV, true>(sm, R, S, z);
                else pass2<0, SB, FIT, kNV>(sm, R, S, z);
            }
            else if (b == 8) pass2<8, SB, FIT, kNV>(sm, R, S, z);
            else if (b == 6) pass2<6, SB, FIT, kNV>(sm, R, S, z);
            else pass2<4, SB, FIT, kNV>(sm, R, S, z);
        }
        if (tid < kD) {
            bar_sync(3, kThreads);
            timed_out = sm.stop != 0;
        }
    }
    if (FIT && MODE != kReadout) {
        __syncthreads();  // the last tile's partial sums are in
        if (!timed_out && tid < kD) fit_finish<SB>(sm, (i + 1) & 1);
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
                if (t < tiles) mbar_wait_bounded(&sm.full[k % kStages], (k / kStages) & 1, p.wait_ns);
            }
        }
        if (sm.flags) atomicOr(p.err, sm.flags);
    }
}

constexpr int kMaxDevices = 64;

template <int KIND, int SB, int MODE, bool FIT>
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
        e = cudaFuncSetAttribute(decode_kernel<KIND, SB, MODE, FIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        sms[dev] = n > 0 ? n : 148;
    }
    const int tiles = io.n * p.H;
    const int grid = tiles < 2 * sms[dev] ? tiles : 2 * sms[dev];
    decode_kernel<KIND, SB, MODE, FIT><<<grid, kThreads, smem, stream>>>(p, io, tiles);
    count_launch();
    return cudaGetLastError();
}

template <int MODE, bool FIT>
cudaError_t launch_fit(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    if (p.scale_bytes == 2)
        return p.kind == STQ_KDA ? launch<STQ_KDA, 2, MODE, FIT>(p, io, stream)
                                 : launch<STQ_GDN, 2, MODE, FIT>(p, io, stream);
    return p.kind == STQ_KDA ? launch<STQ_KDA, 4, MODE, FIT>(p, io, stream)
                             : launch<STQ_GDN, 4, MODE, FIT>(p, io, stream);
}

template <int MODE>
cudaError_t launch_mode(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return p.fit ? launch_fit<MODE, true>(p, io, stream) : launch_fit<MODE, false>(p, io, stream);
}

}  // namespace

cudaError_t launch_decode(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return launch_mode<kFused>(p, io, stream);
}

cudaError_t launch_decode_readout(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return launch_mode<kReadout>(p, io, stream);
}

cudaError_t launch_decode_writeback(const PoolView &p, const DecodeIO &io, cudaStream_t stream)
{
    return launch_mode<kWriteback>(p, io, stream);
}

}  // namespace stq
