// Device-side helpers shared by the SchNet B200 kernels: padded sizes, the
// status word, activation functions, and thin inline-PTX wrappers for the
// sm_100a tensor-core path (tcgen05 MMA with TMEM accumulators, mbarriers).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/schnet.h"

namespace schnet {

// Feature, Gaussian and readout widths are padded to these on the device.
constexpr int FP = 128;   // features (tensor-core M)
constexpr int KP = 64;    // Gaussians (GEMM1 K)
constexpr int HP = 64;    // readout hidden width
constexpr int TILE_E = 128;  // edges per tensor-core tile (GEMM N)

// Accumulators and status shared by all kernels of one context.
struct DevMeta {
    long long n_edges;            // listed edges of the current neighbour list
    unsigned int status;          // SCHNET_FLAG_* bits, sticky until read
    unsigned int pad0;
    unsigned long long step;      // MD step counter (noise stream)
    long long timeout_where;      // diagnostic for bounded waits
};

__device__ __forceinline__ void set_flag(DevMeta* meta, unsigned int bit)
{
    atomicOr(&meta->status, bit);
}

// Programmatic dependent launch (kernels launched with launch_pdl): the next
// kernel on the stream may be scheduled once every CTA of this one has called
// pdl_trigger; pdl_wait blocks until the previous kernel has completed and its
// writes are visible.  Before pdl_wait a kernel touches only data no kernel of
// the step writes (weights, the neighbour build's partitions and edge count, its
// own shared and tensor memory).  Both are no-ops in a kernel launched without
// the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// activations: shifted softplus and its derivative (the logistic function)
// ---------------------------------------------------------------------------
constexpr float LN2F = 0.69314718055994530942f;

__device__ __forceinline__ float ssp(float x)
{
    float t = __expf(-fabsf(x));
    return fmaxf(x, 0.0f) + __logf(1.0f + t) - LN2F;
}

__device__ __forceinline__ float sigmoidf(float x)
{
    float t = __expf(-fabsf(x));
    float r = __fdividef(1.0f, 1.0f + t);
    return x >= 0.0f ? r : t * r;
}

// Single MUFU operations (PTX ex2.approx / lg2.approx, denormals flushed).
constexpr float LOG2EF = 1.44269504088896340736f;

__device__ __forceinline__ float ex2_mufu(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_mufu(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two-wide fp32 arithmetic (sm_100 packed FFMA2 / FMUL2 / FADD2: two lanes of
// ordinary round-to-nearest single precision per instruction).
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// Softplus in base 2 of two values, p = x log2(e).  SHIFT = true: the shifted
// form ssp2(p) = log2(1 + 2^p) - 1 = log2((1 + e^x) / 2) = ssp(x) / ln2, written
// max(p, 0) + log2(1/2 + 2^-|p| / 2); it has no constant offset (ssp2(0) = 0), so
// the products that consume it accumulate no large common term.  SHIFT = false:
// sp2(p) = log2(1 + 2^p) = max(p, 0) + log2(1 + 2^-|p|), which is near 0 rather
// than near -1 for strongly negative x, the better choice for an operand rounded
// once to 16 bits (the -1 then goes into the consumer's bias).  No overflow for
// any p; the logarithm's argument lies in [1/2, 1] or [1, 2].
template <bool SHIFT>
__device__ __forceinline__ float2 sp2x2(float2 p)
{
    const float c = SHIFT ? 0.5f : 1.0f;
    const float2 y = fma2(dup2(c), make_float2(ex2_mufu(-fabsf(p.x)), ex2_mufu(-fabsf(p.y))), dup2(c));
    return add2(make_float2(fmaxf(p.x, 0.0f), fmaxf(p.y, 0.0f)), make_float2(lg2_mufu(y.x), lg2_mufu(y.y)));
}

// 2^x for two arguments x <= 0 on the FMA and integer pipes instead of the MUFU.
// x is clamped at -30 (2^-30 is below half an ulp of 1, so 1 + 2^x rounds the same;
// a NaN is clamped too: non-finite inputs are flagged where the positions enter).
// Cody-Waite reduction x = n + f with n = round(x), found by adding and removing
// 1.5 * 2^23, and f in [-1/2, 1/2]; 2^f by the degree-5 polynomial that
// exp2_fit.py fits (reweighted least squares on Chebyshev nodes; relative error
// <= 2.2e-7 in float32 Horner form); 2^n is added to the exponent field.
__device__ __forceinline__ float2 ex2_fma2(float2 x)
{
    constexpr float RND = 12582912.0f;
    x = make_float2(fmaxf(x.x, -30.0f), fmaxf(x.y, -30.0f));
    const float2 y = add2(x, dup2(RND));
    const float2 n = add2(y, dup2(-RND));
    const float2 f = fma2(n, dup2(-1.0f), x);
    float2 p = fma2(dup2(0.0013276470126584172f), f, dup2(0.009675540961325169f));
    p = fma2(p, f, dup2(0.05550713092088699f));
    p = fma2(p, f, dup2(0.24022120237350464f));
    p = fma2(p, f, dup2(0.6931469440460205f));
    p = fma2(p, f, dup2(1.0000001192092896f));
    const int kx = (__float_as_int(y.x) - __float_as_int(RND)) << 23;
    const int ky = (__float_as_int(y.y) - __float_as_int(RND)) << 23;
    return make_float2(__int_as_float(__float_as_int(p.x) + kx), __int_as_float(__float_as_int(p.y) + ky));
}

// sp2x2 with its exponentials from ex2_fma2 (the logarithms stay on the MUFU)
template <bool SHIFT>
__device__ __forceinline__ float2 sp2x2_fma(float2 p)
{
    const float c = SHIFT ? 0.5f : 1.0f;
    const float2 y = fma2(dup2(c), ex2_fma2(make_float2(-fabsf(p.x), -fabsf(p.y))), dup2(c));
    return add2(make_float2(fmaxf(p.x, 0.0f), fmaxf(p.y, 0.0f)), make_float2(lg2_mufu(y.x), lg2_mufu(y.y)));
}


// ---------------------------------------------------------------------------
// minimum image (single precision, used for distances in the filters)
// ---------------------------------------------------------------------------
struct Box {
    float L[3];
    float invL[3];
    int periodic;
};

__device__ __forceinline__ float3 min_image(float3 v, const Box& b)
{
    if (b.periodic) {
        v.x -= b.L[0] * rintf(v.x * b.invL[0]);
        v.y -= b.L[1] * rintf(v.y * b.invL[1]);
        v.z -= b.L[2] * rintf(v.z * b.invL[2]);
    }
    return v;
}

// Single-precision distance of an edge (minimum image).  Every kernel that
// decides whether an edge lies inside the cutoff uses this one expression, so
// the masking, the filter and the force assembly agree edge by edge.
__device__ __forceinline__ float edge_distance(float4 pi, float4 pj, const Box& b, float3& v)
{
    v = min_image(make_float3(pj.x - pi.x, pj.y - pi.y, pj.z - pi.z), b);
    return sqrtf(v.x * v.x + v.y * v.y + v.z * v.z);
}

// Which of the two edges (i, j) and (j, i) of an unordered pair owns it (carries
// the pair in the half list and its derivative in s_e): (i, j) when i and j differ
// in parity and j > i, or share it and j < i.  Exactly one of the two edges
// qualifies, and each row owns about half of its neighbours wherever it sits in
// the atom order (owning the pairs with j > i would give the early rows nearly all
// of theirs and the late rows almost none), so the rows of the half list and of
// its complement are evenly long.
__device__ __forceinline__ bool owns_pair(int i, int j)
{
    return ((i ^ j) & 1) ? j > i : j < i;
}

// ---------------------------------------------------------------------------
// shared-memory / mbarrier / tcgen05 wrappers (sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after max_iter polls (each poll may itself suspend
// for a hardware-defined slice), returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t max_iter)
{
    for (uint32_t it = 0; it < max_iter; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM allocation by one full warp; the base address lands in *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}


// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM -> 32 registers per thread
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
          "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]),
          "=r"(u[22]), "=r"(u[23]), "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]),
          "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle ("interleaved" core matrices of
// 8 rows x 16 bytes stored as 128 contiguous bytes).  lbo: byte distance
// between core matrices adjacent in K; sbo: adjacent in M/N.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    // base offset 0, absolute LBO mode 0, layout type 0 (no swizzle)
    return d;
}

// Instruction descriptor for kind::f16, dense, f32 accumulate.
// ab_fmt: 0 = f16, 1 = bf16.  b_mn_major: 1 when B is stored MN-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int ab_fmt, int b_mn_major)
{
    return (1u << 4)                          // D format f32
           | ((uint32_t)ab_fmt << 7)          // A format
           | ((uint32_t)ab_fmt << 10)         // B format
           | (0u << 15)                       // A K-major
           | ((uint32_t)b_mn_major << 16)     // B major
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Byte offset of element (mn, k) of a 16-bit operand tile with MN rows,
// no-swizzle core matrices, SBO = 128 B, LBO = MN * 16 B.
__host__ __device__ constexpr uint32_t kmajor_off(int mn, int k, int MN)
{
    return (uint32_t)((k >> 3) * (MN * 16) + mn * 16 + (k & 7) * 2);
}
__host__ __device__ constexpr uint32_t mnmajor_off(int mn, int k, int MN)
{
    return (uint32_t)((k >> 3) * (MN * 16) + (mn >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}


// ---------------------------------------------------------------------------
// tcgen05 helpers shared by the tensor-core kernels
// ---------------------------------------------------------------------------
// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (A read from tensor memory)
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes <- 32 registers per thread
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Row f of one packed weight term (the K-major core-matrix image: K elements
// 8kg .. 8kg+7 of row f are the 16 bytes at kg * 2048 + f * 16), K elements
// 64 * half .. 64 * half + 63, as the 32 registers of one 32-column TMEM store.
__device__ __forceinline__ void weight_row(const uint8_t* __restrict__ term, int f, int half, uint32_t (&v)[32])
{
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(term + (size_t)(half * 8 + q) * (FP * 16) + f * 16));
        v[4 * q] = x.x;
        v[4 * q + 1] = x.y;
        v[4 * q + 2] = x.z;
        v[4 * q + 3] = x.w;
    }
}

// two fp32 values -> packed 16-bit hi pair and lo (residual) pair
template <int FMT>
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo);
template <>
__device__ __forceinline__ void split2<0>(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    __half2 h = __floats2half2_rn(x0, x1);
    float2 hf = __half22float2(h);
    __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}
template <>
__device__ __forceinline__ void split2<1>(float x0, float x1, uint32_t& hi, uint32_t& lo)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// 8 consecutive fp32 values -> one 16-byte hi store and one 16-byte lo store
template <int FMT>
__device__ __forceinline__ void store8(uint8_t* hi_base, uint8_t* lo_base, uint32_t off, const float* v)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) split2<FMT>(v[2 * q], v[2 * q + 1], h[q], l[q]);
    *reinterpret_cast<uint4*>(hi_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo_base + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// 8 consecutive fp32 values -> one 16-byte store of their 16-bit rounding (no lo term)
template <int FMT>
__device__ __forceinline__ void store8_hi(uint8_t* hi_base, uint32_t off, const float* v)
{
    uint32_t h[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (FMT == 0) {
            __half2 x = __floats2half2_rn(v[2 * q], v[2 * q + 1]);
            h[q] = *reinterpret_cast<uint32_t*>(&x);
        } else {
            __nv_bfloat162 x = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            h[q] = *reinterpret_cast<uint32_t*>(&x);
        }
    }
    *reinterpret_cast<uint4*>(hi_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
}

// two fp32 values -> packed 16-bit hi pair and the NEGATED residual pair: hi - x
// (exact in fp32, since it is the rounding error of hi) by the mixed-precision
// subtract of the 16-bit hi and the fp32 x, then rounded once to 16 bits -- the
// same bits as -RN16(x - hi), without converting hi back to fp32.  The MMAs that
// read this term negate their B operand (instruction-descriptor bit 14).
template <int FMT>
__device__ __forceinline__ void split2_neg(float x0, float x1, uint32_t& hi, uint32_t& nlo);
template <>
__device__ __forceinline__ void split2_neg<0>(float x0, float x1, uint32_t& hi, uint32_t& nlo)
{
    asm("{\n\t.reg .b16 l, u;\n\t.reg .f32 d0, d1;\n\t"
        "cvt.rn.f16x2.f32 %0, %3, %2;\n\t"
        "mov.b32 {l, u}, %0;\n\t"
        "sub.rn.f32.f16 d0, l, %2;\n\t"
        "sub.rn.f32.f16 d1, u, %3;\n\t"
        "cvt.rn.f16x2.f32 %1, d1, d0;\n\t}"
        : "=r"(hi), "=r"(nlo)
        : "f"(x0), "f"(x1));
}
template <>
__device__ __forceinline__ void split2_neg<1>(float x0, float x1, uint32_t& hi, uint32_t& nlo)
{
    asm("{\n\t.reg .b16 l, u;\n\t.reg .f32 d0, d1;\n\t"
        "cvt.rn.bf16x2.f32 %0, %3, %2;\n\t"
        "mov.b32 {l, u}, %0;\n\t"
        "sub.rn.f32.bf16 d0, l, %2;\n\t"
        "sub.rn.f32.bf16 d1, u, %3;\n\t"
        "cvt.rn.bf16x2.f32 %1, d1, d0;\n\t}"
        : "=r"(hi), "=r"(nlo)
        : "f"(x0), "f"(x1));
}

// instruction-descriptor bit of a negated B operand (the negated-residual terms)
constexpr uint32_t IDESC_NEG_B = 1u << 14;

// activation operand: hi and negated-residual pair (NX = 2), or the 16-bit rounding
// alone (NX = 1)
template <int FMT, int NX>
__device__ __forceinline__ void store8_act(uint8_t* hi_base, uint8_t* lo_base, uint32_t off, const float* v)
{
    if (NX == 2) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) split2_neg<FMT>(v[2 * q], v[2 * q + 1], h[q], l[q]);
        *reinterpret_cast<uint4*>(hi_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lo_base + off) = make_uint4(l[0], l[1], l[2], l[3]);
    } else {
        store8_hi<FMT>(hi_base, off, v);
    }
}


// 32 lanes x 16 columns of TMEM -> 16 registers per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16])
{
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}

}  // namespace schnet
