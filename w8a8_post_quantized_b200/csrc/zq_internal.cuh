// zq_internal.cuh -- shared device helpers and host launcher declarations
// for the sm_100a W8A8 library.  Inline PTX for mbarrier, TMA (bulk tensor
// copies), and the 5th-generation tensor core (tcgen05: TMEM allocation,
// MMA, commit, TMEM loads).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include "zq.h"

namespace zq {

// ----------------------------------------------------------------- general

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bf16 bit pattern -> fp32 (exact)
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp32 pair -> two bf16 (round to nearest even) packed low|high
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// GeLU(x) = x * Phi(x), Phi the standard normal CDF, Phi(x) = (1 + erf(x/sqrt2))/2.
// Branch-free: with u = |x|/sqrt2, the complementary error function is taken
// from the rational approximation of Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (after Hastings):
//   erfc(u) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-u^2),
//   t = 1 / (1 + p u),  |error| <= 1.5e-7 for u >= 0;
// Phi(-|x|) = erfc(u)/2 and Phi(|x|) = 1 - Phi(-|x|).  The coefficients below
// are the published ones halved (folding the 1/2).
__device__ __forceinline__ float gelu_f(float x) {
    constexpr float kP = 0.3275911f;
    constexpr float kA1 = 0.5f * 0.254829592f, kA2 = 0.5f * -0.284496736f, kA3 = 0.5f * 1.421413741f,
                    kA4 = 0.5f * -1.453152027f, kA5 = 0.5f * 1.061405429f;
    const float u = fabsf(x) * 0.70710678118654752f;
    float t, e;
    // hardware reciprocal and base-2 exponential (relative error about 2^-22):
    // far below the 1.5e-7 of the approximation itself.  Flushing subnormals
    // is harmless: the reciprocal's argument is >= 1 and an exponential below
    // 2^-126 leaves Phi(-|x|) far under one ulp of the result.
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(kP, u, 1.0f)));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x * x * -0.72134752044448170f));  // exp(-x^2/2)
    const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, kA5, kA4), kA3), kA2), kA1);
    const float lower = poly * e;                             // Phi(-|x|)
    return x * (x >= 0.0f ? 1.0f - lower : lower);
}

// Symmetric code: clamp(rint(y * inv), -127, 127).  The product is a single
// fp32 rounding (no contraction); rintf rounds ties to even.
__device__ __forceinline__ int quant_code(float y, float inv) {
    float r = rintf(__fmul_rn(y, inv));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return __float2int_rz(r);
}

__device__ __forceinline__ uint32_t pack_i8x4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
           ((uint32_t)(d & 0xFF) << 24);
}

// scale = absmax/127 and inv = 127/absmax as IEEE-rounded fp32 divisions;
// an all-zero span gets inv = 0 so every code is 0 and the scale is 0.
__device__ __forceinline__ void absmax_scales(float amax, float& scale, float& inv) {
    scale = __fdiv_rn(amax, 127.0f);
    inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait limit for every device-side wait (ns).  A correct kernel waits
// microseconds; the limit only turns a logic error into an error status.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait on phase `parity` of `bar`.  Gives up when the CTA-wide abort
// flag is raised by another role, or after kWaitLimitNs, in which case it
// records `site` in the device status word and raises the abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (abort_flag && *abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicCAS(status, 0, site);
                if (abort_flag) *abort_flag = 1;
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared, completion counted in bytes on
// `bar`.  c0 is the innermost (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0,
                                            int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// 1-D bulk copy global -> shared (contiguous bytes), completion counted on
// `bar`.  Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Round to nearest even and saturate to [-128, 127] in one conversion.  For
// |y| <= absmax and inv = fp32(127/absmax), |y*inv| <= 127*(1+2^-24), so the
// result always lies in [-127, 127] and equals clamp(rint(y*inv), -127, 127).
__device__ __forceinline__ uint32_t quant_code_sat(float y, float inv) {
    uint32_t r;
    asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(r) : "f"(__fmul_rn(y, inv)));
    return r & 0xFFu;
}

// ------------------------------------------------- packed fp32 pairs (sm_100)
// A pair of fp32 values in one 64-bit register; add/sub/mul/fma on the pair
// issue as one instruction (each lane is still IEEE round-to-nearest).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ uint64_t f2_splat(float v) { return f2_pack(v, v); }
// two 32-bit words as one 64-bit register pair, lo first
__device__ __forceinline__ uint64_t u2_pack(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

// GeLU of a pair of values in packed fp32 arithmetic, the approximation of
// gelu_f rearranged to need no select: with a = |x| and L = Phi(-a),
//   gelu(x) = x * Phi(x) = x/2 + a * (1/2 - L)
// (x >= 0: x/2 + x/2 - x L = x - x L;  x < 0: x/2 - x/2 + x L = x Phi(x)).  L is
// the Abramowitz & Stegun 7.1.26 form t P(t) exp(-a^2/2) / 2 with
// t = 1/(1 + p a/sqrt2); the coefficients enter negated and halved (Q = -P/2)
// so that 1/2 - L = fma(t Q(t), exp(-a^2/2), 1/2) and the last step is one
// fused multiply-add.  For x < 0 the two halves cancel inside that FMA, which
// leaves an absolute error of about |x| 2^-25 (far below the approximation's
// 1.5e-7 * |x|).
__device__ __forceinline__ uint64_t gelu2(uint64_t x2) {
    constexpr float kPs = 0.3275911f * 0.70710678118654752f;
    constexpr float kB1 = -0.5f * 0.254829592f, kB2 = -0.5f * -0.284496736f, kB3 = -0.5f * 1.421413741f,
                    kB4 = -0.5f * -1.453152027f, kB5 = -0.5f * 1.061405429f;
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const uint64_t a2 = f2_pack(fabsf(x0), fabsf(x1));
    float d0, d1, q0, q1, t0, t1, e0, e1;
    f2_unpack(f2_fma(a2, f2_splat(kPs), f2_splat(1.0f)), d0, d1);
    f2_unpack(f2_mul(f2_mul(a2, f2_splat(-0.72134752044448170f)), a2), q0, q1);  // -a^2/2 * log2(e)
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(d0));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(d1));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(q0));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(q1));
    const uint64_t t2 = f2_pack(t0, t1);
    uint64_t h = f2_fma(t2, f2_splat(kB5), f2_splat(kB4));
    h = f2_fma(t2, h, f2_splat(kB3));
    h = f2_fma(t2, h, f2_splat(kB2));
    h = f2_fma(t2, h, f2_splat(kB1));
    const uint64_t w = f2_fma(f2_mul(h, t2), f2_pack(e0, e1), f2_splat(0.5f));  // 1/2 - L
    return f2_fma(a2, w, f2_mul(x2, f2_splat(0.5f)));
}

// 32 int32 accumulators -> 16 packed fp32 pairs, rounded to nearest (exact
// while |acc| < 2^24, which holds for any K <= 1040).  A variant that avoids
// cvt -- the word 0x4B400000 + acc read as the float 1.5*2^23 + acc, with a
// per-chunk range check -- measured slower on B200: the check costs more
// issue slots than the conversion.
__device__ __forceinline__ void acc32_to_f2(const uint32_t (&v)[32], uint64_t (&f)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = f2_pack((float)(int)v[2 * i], (float)(int)v[2 * i + 1]);
}

// One 32-column chunk of one output row, dequantized in packed pairs:
//   y[j] = (row_scale * sc[j]) * acc[j] + bias[j]   (+ GeLU),
// one fused multiply-add per value after the exact int32 -> fp32 conversion.
// UNI: all 32 columns share one scale (sc[0]).  Bias from shared memory
// (bias_s) or, when bias_s is null, from global memory through L1 (bias_g,
// 16-byte loads; columns at or past nb read 0; bias_g may then be null).
template <bool GELU, bool UNI>
__device__ __forceinline__ void dequant_chunk(uint32_t (&v)[32], float row_scale, const float* sc,
                                              const float* bias_s, const float* bias_g, int nb,
                                              uint64_t (&f)[16]) {
    acc32_to_f2(v, f);
    const uint64_t rs2 = f2_splat(row_scale);
    const uint64_t a_uni = f2_splat(row_scale * sc[0]);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint64_t b01, b23;
        if (bias_s) {
            b01 = *reinterpret_cast<const uint64_t*>(bias_s + 4 * q);
            b23 = *reinterpret_cast<const uint64_t*>(bias_s + 4 * q + 2);
        } else {
            const float4 t4 = 4 * q < nb ? __ldg(reinterpret_cast<const float4*>(bias_g) + q)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
            b01 = f2_pack(t4.x, t4.y);
            b23 = f2_pack(t4.z, t4.w);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = 2 * q + e;
            const uint64_t a2 = UNI ? a_uni : f2_mul(rs2, *reinterpret_cast<const uint64_t*>(sc + 2 * i));
            uint64_t t = f2_fma(a2, f[i], e ? b23 : b01);
            if (GELU) t = gelu2(t);
            f[i] = t;
        }
    }
}

// The same with the column factors held across the warp: lane l carries the
// weight-group scale (ca) and the bias (cb, 0 without bias) of column l of the
// chunk; they reach every lane by shuffles (no shared-memory staging).
template <bool GELU, bool UNI>
__device__ __forceinline__ void dequant_chunk_lanes(uint32_t (&v)[32], float row_scale, float ca, float cb,
                                                    uint64_t (&f)[16]) {
    acc32_to_f2(v, f);
    const uint64_t rs2 = f2_splat(row_scale);
    const uint64_t a_uni = f2_splat(row_scale * __shfl_sync(0xFFFFFFFFu, ca, 0));
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint64_t a2 = UNI ? a_uni
                                : f2_mul(rs2, f2_pack(__shfl_sync(0xFFFFFFFFu, ca, 2 * i),
                                                      __shfl_sync(0xFFFFFFFFu, ca, 2 * i + 1)));
        const uint64_t b2 = f2_pack(__shfl_sync(0xFFFFFFFFu, cb, 2 * i), __shfl_sync(0xFFFFFFFFu, cb, 2 * i + 1));
        uint64_t t = f2_fma(a2, f[i], b2);
        if (GELU) t = gelu2(t);
        f[i] = t;
    }
}

// fp16 halves of a 32-bit word (low half first), as floats.
__device__ __forceinline__ float half_lo(uint32_t w) {
    float f;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(f) : "r"(w));
    return f;
}
__device__ __forceinline__ float half_hi(uint32_t w) {
    float f;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, hi;\n\t}" : "=f"(f) : "r"(w));
    return f;
}

// dequant_chunk_lanes plus the LLM.int8() outlier part: before bias and
// activation each column gains sum_k xo[k] * wo[column][k] (the decomposed
// columns' fp16 values, exact products accumulated in fp32); the warp's
// outlier weights sit transposed in shared memory, box[k * 32 + column].
template <bool GELU, bool UNI>
__device__ __forceinline__ void dequant_chunk_lanes_outl(uint32_t (&v)[32], float row_scale, float ca, float cb,
                                                         const float (&xo)[8], const float* box, uint64_t (&f)[16]) {
    acc32_to_f2(v, f);
    const uint64_t rs2 = f2_splat(row_scale);
    const uint64_t a_uni = f2_splat(row_scale * __shfl_sync(0xFFFFFFFFu, ca, 0));
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint64_t a2 = UNI ? a_uni
                                : f2_mul(rs2, f2_pack(__shfl_sync(0xFFFFFFFFu, ca, 2 * i),
                                                      __shfl_sync(0xFFFFFFFFu, ca, 2 * i + 1)));
        uint64_t o2 = f2_pack(__shfl_sync(0xFFFFFFFFu, cb, 2 * i), __shfl_sync(0xFFFFFFFFu, cb, 2 * i + 1));
#pragma unroll
        for (int k = 0; k < 8; ++k)
            o2 = f2_fma(f2_splat(xo[k]), *reinterpret_cast<const uint64_t*>(box + k * 32 + 2 * i), o2);
        uint64_t t = f2_fma(a2, f[i], o2);
        if (GELU) t = gelu2(t);
        f[i] = t;
    }
}

// Codes of four fp32 values packed little-endian into one word.
// t = fl(y * inv) as a packed multiply; then fl(t + 1.5*2^23) (a scalar add
// with explicit round-to-nearest, which is never contracted with the multiply)
// holds rint(t), ties to even, in its low mantissa bits; the low byte is the
// two's-complement code.  For |y| <= absmax, |t| <= 127*(1+2^-24), so no clamp
// is ever active and the code equals clamp(rint(fl(y*inv)), -127, 127).
// (A packed add here would be fused with the packed multiply into one FMA,
// rounding once instead of twice.)
__device__ __forceinline__ uint32_t quant4_packed(uint64_t y01, uint64_t y23, uint64_t inv2) {
    const float magic = 12582912.0f;  // 1.5 * 2^23
    float t0, t1, t2, t3;
    f2_unpack(f2_mul(y01, inv2), t0, t1);
    f2_unpack(f2_mul(y23, inv2), t2, t3);
    const uint32_t c0 = __float_as_uint(__fadd_rn(t0, magic));
    const uint32_t c1 = __float_as_uint(__fadd_rn(t1, magic));
    const uint32_t c2 = __float_as_uint(__fadd_rn(t2, magic));
    const uint32_t c3 = __float_as_uint(__fadd_rn(t3, magic));
    return __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
}

// Codes of four values with a single rounding: rint(y*inv) computed as one
// fused multiply-add with the 1.5*2^23 constant.  It differs from the
// two-rounding form above only when y*inv lies within half an fp32 ulp of a
// tie; used where y is itself an fp32 approximation (LayerNorm, GeLU) and the
// codes are compared within a tolerance, never on the bit-exact paths.
__device__ __forceinline__ uint32_t quant4_packed_fused(uint64_t y01, uint64_t y23, uint64_t inv2) {
    const uint64_t magic = 0x4B4000004B400000ull;  // (1.5*2^23, 1.5*2^23)
    const uint64_t m01 = f2_fma(y01, inv2, magic);
    const uint64_t m23 = f2_fma(y23, inv2, magic);
    return __byte_perm(__byte_perm((uint32_t)m01, (uint32_t)(m01 >> 32), 0x0040),
                       __byte_perm((uint32_t)m23, (uint32_t)(m23 >> 32), 0x0040), 0x5410);
}

// 2-D tiled bulk tensor store shared -> global (one thread), tracked as a
// bulk async-group of the issuing thread.  Coordinates are never negative;
// elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// until this thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// until at most one of this thread's bulk store groups is still reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// until this thread's bulk stores have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Row `r` (0..31) of a 32-row staging box whose rows are RB bytes (32, 64 or
// 128), written as RB/16 16-byte chunks at the positions the TMA swizzle of
// the same width expects (32B, 64B, 128B modes): chunk j lands at
// j ^ ((r >> s) & (RB/16 - 1)) with s = 2, 1, 0.  Eight consecutive rows then
// cover all 32 banks, so the warp's writes are conflict-free.
template <int RB>
__device__ __forceinline__ void stage_row_swizzled(uint8_t* box, int r, const uint32_t* words) {
    constexpr int NCH = RB / 16;
    constexpr int SH = RB == 128 ? 0 : RB == 64 ? 1 : 2;
    uint4* row = reinterpret_cast<uint4*>(box + r * RB);
#pragma unroll
    for (int j = 0; j < NCH; ++j)
        row[j ^ ((r >> SH) & (NCH - 1))] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle (8-row x 128-byte atoms, 1024 bytes between 8-row groups).
// Fields: start address >> 4 (bits 0-13), leading byte offset >> 4 (16-29,
// unused for this layout), stride byte offset >> 4 (32-45), descriptor
// version 1 (46-47), layout type 2 = 128B swizzle (61-63).
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::i8: D = s32 (bits 4-5 = 2), A and B signed
// 8-bit (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, one thread issues.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// lane (base lane + i), columns col .. col+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ int4 ld_cluster_v4(uint32_t cluster_addr) {
    int4 v;
    asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// shared::cta address -> the same offset in the shared memory of cluster CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// Programmatic dependent launch.  griddep_wait: block until every grid this
// one depends on has completed and its memory is visible (immediate when the
// launch has no such dependency).  griddep_launch_dependents: this CTA no
// longer holds back the launch of the next grid in the stream; that grid's
// CTAs then take free SMs and wait in griddep_wait, so its launch latency and
// prologue overlap this grid's tail.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Asynchronous 4-byte store into a cluster peer's shared memory that counts
// its bytes on the peer's mbarrier (complete-tx); both addresses from mapa.
__device__ __forceinline__ void st_async_u32(uint32_t cluster_addr, uint32_t v, uint32_t cluster_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(cluster_addr),
                 "r"(v), "r"(cluster_bar)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait with cluster-scope acquire (data written by peer CTAs)
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  int* status, int site) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait_acq_cluster(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (abort_flag && *abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicCAS(status, 0, site);
                if (abort_flag) *abort_flag = 1;
                return false;
            }
        }
    }
}
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
// every thread of every CTA of the cluster
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

}  // namespace zq

// ------------------------------------------------------------- host side

namespace zq {

// Per-device cached facts (SM count, compute capability) and the device
// address of the library's status word.
struct DeviceInfo {
    int sm_count;
    int major, minor;
    int* status_word;  // device pointer
};
int device_info(DeviceInfo* out);  // returns zq_status

void set_cuda_error(cudaError_t e);
void count_launch();  // every kernel launch goes through this
// Programmatic dependent launch for the hot-path kernels: fills `attr` with
// the stream-serialization attribute (returns 1) unless ZQ_NO_PDL is set in
// the environment (returns 0).  Kernels launched with it call griddep_wait()
// before touching global memory.
int pdl_attr(cudaLaunchAttribute& attr);
int cuda_status(cudaError_t e);  // ZQ_OK or ZQ_ERR_CUDA (and records the text)
// Guards the launchers' per-device caches (kernel attributes set, occupancy
// and register counts queried once per device), which several host threads
// may fill at the same time on their first calls.
std::mutex& launch_cache_mutex();

// launchers (no validation; the C ABI validates)
int launch_quantize_weights(const float* W, int64_t N, int64_t K, int64_t G, int8_t* Wq,
                            float* s_grp, const DeviceInfo& di, cudaStream_t st);
int launch_ln_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                    const float* beta, float eps, int8_t* q, float* s_tok, const DeviceInfo& di,
                    cudaStream_t st);
int launch_act_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* bias, int act,
                     int8_t* q, float* s_tok, const DeviceInfo& di, cudaStream_t st);
// Pipelined row quantizers (bulk copies into a shared-memory ring); return
// ZQ_ERR_SHAPE when H is outside their range so the caller can fall back.
int launch_rowq_pipe(const void* x, int x_dtype, int64_t T, int64_t H, bool ln, const float* gamma,
                     const float* beta, float eps, const float* bias, int act, int8_t* q,
                     float* s_tok, const DeviceInfo& di, cudaStream_t st);
int launch_requant_rows(const float* h, int64_t T, int64_t N, const uint32_t* amax_bits, int8_t* q,
                        float* s_tok, const DeviceInfo& di, cudaStream_t st);
int launch_llmint8_select(const float* amax, int64_t K, float threshold, const float* gamma, const float* beta,
                          int32_t* idx, int32_t* count, float* gamma_m, float* beta_m, cudaStream_t st);
int launch_llmint8_outlier_act(const void* x, int x_dtype, int64_t T, int64_t K, const float* gamma,
                               const float* beta, float eps, const int32_t* idx, const int32_t* count, uint16_t* xo,
                               cudaStream_t st);
int launch_llmint8_outlier_weights(const float* W, int64_t N, int64_t K, const int32_t* idx, const int32_t* count,
                                   uint16_t* wo, cudaStream_t st);
int launch_smooth_calibrate(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                            const float* beta, float eps, float* amax, const DeviceInfo& di, cudaStream_t st);
int launch_smooth_weights(const float* W, int64_t N, int64_t K, const float* amax, float alpha, const float* gamma,
                          const float* beta, float* W_out, float* gamma_out, float* beta_out, float* s,
                          const DeviceInfo& di, cudaStream_t st);

struct LinearArgs {
    const int8_t* xq;
    const float* s_tok;
    int64_t T, K;
    const int8_t* Wq;
    const float* s_grp;
    int64_t N, G;
    const float* bias;
    int act, out_kind;
    void* y;
    float* s_tok_out;   // REQUANT: new per-token scales [T]
    float* h_ws;        // REQUANT (scratch path): fp32 [T, N]
    uint32_t* amax_ws;  // REQUANT (scratch path): [T] absmax bit patterns
};
int launch_w8a8_gemm(const LinearArgs& a, const DeviceInfo& di, cudaStream_t st);
int launch_w8a8_gemm_outliers(const LinearArgs& a, const uint16_t* xo, const uint16_t* wo, const DeviceInfo& di,
                              cudaStream_t st);
// Few-token linear (T <= 64; f32, bf16 or raw int32 output; weights on the
// MMA's M side) with the (weight tile, k-block) iterations in equal
// contiguous ranges, one persistent CTA per SM.  A tile that a range boundary
// cuts is summed from int32 partials in `ws` (decode_sk_ws_bytes(sm_count)
// bytes, 16-byte aligned), with one ready flag per CTA zeroed by a small
// kernel launched first.  ZQ_ERR_SHAPE: not covered; ZQ_ERR_WORKSPACE: ws
// missing or too small (nothing launched); the caller then takes
// launch_w8a8_gemm.  decode_even_applies: whether the shape takes this route
// on a device with `sms` SMs (ZQ_EVEN_SPLIT overrides the choice).
size_t decode_sk_ws_bytes(int sms);
bool decode_even_applies(int64_t T, int64_t K, int64_t N, int sms);
int launch_w8a8_decode_sk(const LinearArgs& a, void* ws, size_t ws_bytes, const DeviceInfo& di, cudaStream_t st);
// 0 = the choice above, 1 = never split evenly, 2 = always when the kernel
// covers the shape (environment variable ZQ_EVEN_SPLIT = off | on, read on
// every call; for measurements and tests).
int even_split_mode();
// Requantizing linear with the per-token absmax exchanged between the CTAs of
// a thread-block cluster (no scratch).  ZQ_ERR_SHAPE: shape not covered (the
// caller then uses the scratch path).
int launch_w8a8_requant_cluster(const LinearArgs& a, const DeviceInfo& di, cudaStream_t st);
// Requantizing linear for rows of any width in one persistent kernel: the
// per-token absmax goes through global atomics and per-row-block arrival
// counters in `scratch` (requant_grid_scratch_bytes(T) bytes, zeroed by the
// launcher).  ZQ_ERR_SHAPE: shape not covered (T <= 64, or more column tiles
// per row than co-resident CTAs).
// ZQ_ERR_WORKSPACE: the kernel applies but scratch_bytes is too small
// (checked before anything is launched).
size_t requant_grid_scratch_bytes(int64_t T);
int launch_w8a8_requant_grid(const LinearArgs& a, uint32_t* scratch, size_t scratch_bytes, const DeviceInfo& di,
                             cudaStream_t st);
// Scratch of the requantizing linear: the bytes the route for this shape
// needs on a device with `sms` SMs (sms <= 0: unknown, assume the scratch
// route), and the bytes of the scratch route (fp32 output + absmax words).
size_t requant_ws_bytes(int64_t T, int64_t N, int sms);
size_t requant_scratch_route_bytes(int64_t T, int64_t N);
// The requantizing linear through its routes (cluster kernel, grid kernel,
// scratch route) with `ws` as scratch; returns err_small, having launched
// nothing, when the route the shape takes needs more than ws_bytes.
int run_requant(const LinearArgs& a, void* ws, size_t ws_bytes, int err_small, const DeviceInfo& di,
                cudaStream_t st);
// Which requantizing route zq_w8a8_linear takes: 0 = automatic, 1 = cluster
// kernel only, 2 = grid kernel only, 3 = scratch route (environment variable
// ZQ_REQUANT_ROUTE = cluster | grid | scratch; for measurements).
int requant_route();
// int8 matrix [rows, K] as a TMA tensor: box 128 bytes of K x box_rows rows,
// 128-byte swizzle, out-of-range elements read as 0.
int make_tmap_i8(CUtensorMap* tm, const void* ptr, int64_t rows, int64_t K, int box_rows);
// Output matrix [rows, cols] of `esize`-byte elements as a TMA store target:
// box 32 columns x 32 rows, swizzle matching the 32*esize-byte box rows.
int make_tmap_out(CUtensorMap* tm, void* ptr, int64_t rows, int64_t cols, int esize);

}  // namespace zq
