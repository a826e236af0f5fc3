// common.cuh -- small device helpers shared by the kernels of this library (sm_100a only).
//
// Hand-written inline PTX for: mbarriers, bulk (TMA) copies, acquire/release flags, the
// global timer used to bound every wait, bf16 packing, and approximate ex2/rcp.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

#define RAT_DEVICE __device__ __forceinline__

namespace rat {

// ------------------------------------------------------------------------------ elements
struct f32x4 { float v[4]; };

RAT_DEVICE float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
RAT_DEVICE float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Round two floats to bf16 (nearest-even) and pack them, lo in bits 0..15.
RAT_DEVICE uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------------------------------------ float pairs
// Two float32 lanes in one 64-bit register pair, for the packed f32x2 arithmetic of sm_100
// (one instruction per pair, IEEE round-to-nearest like the scalar forms).
typedef unsigned long long f2_t;
RAT_DEVICE f2_t f2(float lo, float hi) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
RAT_DEVICE float f2lo(f2_t v) {
    float lo;
    asm("{\n .reg .f32 t;\n mov.b64 {%0, t}, %1;\n}" : "=f"(lo) : "l"(v));
    return lo;
}
RAT_DEVICE float f2hi(f2_t v) {
    float hi;
    asm("{\n .reg .f32 t;\n mov.b64 {t, %0}, %1;\n}" : "=f"(hi) : "l"(v));
    return hi;
}
RAT_DEVICE f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
RAT_DEVICE f2_t f2_mul(f2_t a, f2_t b) {
    f2_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
RAT_DEVICE f2_t f2_add(f2_t a, f2_t b) {
    f2_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// bf16 pair (low element in bits 0..15) -> float pair, and back (round to nearest even)
// max(a, b, c) in one instruction (three-input max.f32, sm_100).
RAT_DEVICE float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
RAT_DEVICE f2_t f2_from_bf16x2(uint32_t u) { return f2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u)); }
RAT_DEVICE uint32_t f2_to_bf16x2(f2_t v) { return pack_bf16(f2lo(v), f2hi(v)); }

// ------------------------------------------------------------------------------ rows
// A lane's two channel pairs of one row: pair 0 at channels (2l, 2l+1), pair 1 at
// (2l + d/2, 2l+1 + d/2), as float pairs.
template <typename E> struct Lane;
template <> struct Lane<float> {
    template <int HALFB>
    static RAT_DEVICE void load(const uint8_t *row, int l, f2_t *x) {
        const uint2 a = *reinterpret_cast<const uint2 *>(row + 8 * l);
        const uint2 c = *reinterpret_cast<const uint2 *>(row + HALFB + 8 * l);
        x[0] = f2(__uint_as_float(a.x), __uint_as_float(a.y));
        x[1] = f2(__uint_as_float(c.x), __uint_as_float(c.y));
    }
    template <int HALFB>
    static RAT_DEVICE void store(uint8_t *row, int l, const f2_t *x) {
        *reinterpret_cast<uint2 *>(row + 8 * l) = make_uint2(__float_as_uint(f2lo(x[0])), __float_as_uint(f2hi(x[0])));
        *reinterpret_cast<uint2 *>(row + HALFB + 8 * l) = make_uint2(__float_as_uint(f2lo(x[1])), __float_as_uint(f2hi(x[1])));
    }
};
template <> struct Lane<__nv_bfloat16> {
    template <int HALFB>
    static RAT_DEVICE void load(const uint8_t *row, int l, f2_t *x) {
        x[0] = f2_from_bf16x2(*reinterpret_cast<const uint32_t *>(row + 4 * l));
        x[1] = f2_from_bf16x2(*reinterpret_cast<const uint32_t *>(row + HALFB + 4 * l));
    }
    template <int HALFB>
    static RAT_DEVICE void store(uint8_t *row, int l, const f2_t *x) {
        *reinterpret_cast<uint32_t *>(row + 4 * l) = f2_to_bf16x2(x[0]);
        *reinterpret_cast<uint32_t *>(row + HALFB + 4 * l) = f2_to_bf16x2(x[1]);
    }
};

// CPL consecutive channels of one row per lane (the CUDA-core attention kernels), as floats.
template <typename E, int CPL> struct RowIO;
template <> struct RowIO<float, 2> {
    static RAT_DEVICE void load(const void *p, float *x) {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
        x[0] = v.x; x[1] = v.y;
    }
    static RAT_DEVICE void store(void *p, const float *x) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};
template <> struct RowIO<float, 4> {
    static RAT_DEVICE void load(const void *p, float *x) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static RAT_DEVICE void store(void *p, const float *x) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <> struct RowIO<__nv_bfloat16, 2> {
    static RAT_DEVICE void load(const void *p, float *x) {
        const uint32_t u = __ldg(reinterpret_cast<const unsigned int *>(p));
        x[0] = bf16_lo(u); x[1] = bf16_hi(u);
    }
    static RAT_DEVICE void store(void *p, const float *x) {
        *reinterpret_cast<uint32_t *>(p) = pack_bf16(x[0], x[1]);
    }
};
template <> struct RowIO<__nv_bfloat16, 4> {
    static RAT_DEVICE void load(const void *p, float *x) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    }
    static RAT_DEVICE void store(void *p, const float *x) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
    }
};

RAT_DEVICE float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ------------------------------------------------------------------------------ math
// 2^x and 1/x from the special-function unit (PTX ex2.approx / rcp.approx, flush-to-zero).
RAT_DEVICE float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
RAT_DEVICE float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Forget gate from its logit: g = 1/(1+e^{-a}) and 1-g = e^{-a}/(1+e^{-a}).
// For a -> -inf, e^{-a} = inf, g = 0 and the product inf*0 is NaN: fminf maps it to 1 exactly,
// and also caps rounding of e*g slightly above 1.  For a -> +inf, e = 0, g = 1, 1-g = 0.
RAT_DEVICE void forget_gate(float a, float &g, float &omg) {
    const float kLog2e = 1.4426950408889634f;
    float e = ex2_approx(-a * kLog2e);
    g = rcp_approx(1.0f + e);
    omg = fminf(e * g, 1.0f);
}

// cos/sin of pos * theta for RoPE.  The angle is formed in float64 and reduced by 2*pi with a
// two-term (Cody-Waite) constant, so positions up to 2^31 keep full single-precision accuracy;
// the reduced angle in [-pi, pi] goes to the single-precision sincosf.
RAT_DEVICE void rope_cs(long long pos, double theta, float &c, float &s) {
    const double kTwoPiHi = 6.283185307179586;          // nearest double to 2*pi
    const double kTwoPiLo = 2.4492935982947064e-16;     // 2*pi - kTwoPiHi
    const double kInvTwoPi = 0.15915494309189535;
    const double ang = (double)pos * theta;
    const double n = rint(ang * kInvTwoPi);
    double r = fma(-n, kTwoPiHi, ang);
    r = fma(-n, kTwoPiLo, r);
    sincosf((float)r, &s, &c);
}

// Same with a float32 angle, for positions where pos * theta stays below 2^13 rad: the float32
// product is then within 2.5e-4 rad of the exact angle, reduced by a two-term float 2*pi, and the
// special-function-unit sincos is accurate to ~1e-6 on [-pi, pi].  Used only for bf16 outputs.
RAT_DEVICE void rope_cs_f32(int pos, float theta, float &c, float &s) {
    const float kTwoPiHi = 6.28318548f, kTwoPiLo = -1.7484555e-7f;   // 2*pi = hi + lo
    const float ang = (float)pos * theta;
    const float n = rintf(ang * 0.159154943f);
    float r = fmaf(-n, kTwoPiHi, ang);
    r = fmaf(-n, kTwoPiLo, r);
    __sincosf(r, &s, &c);
}

// Forget gate of a pair of logits: g = sigmoid(a) = 1 / (1 + 2^(-a log2 e)).  The
// complement is formed by gate_complement2 as 1 - g: exact for g >= 1/2 (Sterbenz), within
// 2^-25 absolute below, and exactly 0 or 1 at the saturated gates.
RAT_DEVICE f2_t forget_gate2(f2_t a) {
    const f2_t kNegLog2e = f2(-1.4426950408889634f, -1.4426950408889634f);
    const f2_t kOne = f2(1.f, 1.f);
    const f2_t x = f2_mul(a, kNegLog2e);
    const f2_t e = f2(ex2_approx(f2lo(x)), ex2_approx(f2hi(x)));
    const f2_t y = f2_add(e, kOne);
    return f2(rcp_approx(f2lo(y)), rcp_approx(f2hi(y)));
}
RAT_DEVICE f2_t gate_complement2(f2_t g) { return f2_fma(g, f2(-1.f, -1.f), f2(1.f, 1.f)); }

// ------------------------------------------------------------------------------ memory order
RAT_DEVICE uint64_t ld_relaxed_gpu_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
RAT_DEVICE void st_relaxed_gpu_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}
RAT_DEVICE uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
RAT_DEVICE void st_release_gpu(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
RAT_DEVICE uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record the first device-side error of a launch in the workspace header.
RAT_DEVICE void record_error(WsHeader *hdr, int code, uint32_t detail) {
    if (hdr && atomicCAS(&hdr->error, 0, code) == 0) hdr->detail = detail;
}

// ------------------------------------------------------------------------------ smem / mbarrier
RAT_DEVICE uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

RAT_DEVICE void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
RAT_DEVICE void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
RAT_DEVICE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
RAT_DEVICE void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
RAT_DEVICE bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier, for at most kWaitLimitNs.  Returns false (and
// records RAT_ERR_TIMEOUT when hdr is given) if the wait ran out.
RAT_DEVICE bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, WsHeader *hdr, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    uint32_t tries = 0;
    while (!mbar_try_wait(bar, parity)) {
        if ((++tries & 15u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) {
            if (hdr) record_error(hdr, RAT_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// One-dimensional bulk copy global -> shared (the untiled TMA path), completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
RAT_DEVICE void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

RAT_DEVICE void ld_shared_v4(const void *p, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(smem_u32(p)));
}
RAT_DEVICE void ld_shared_v2(const void *p, uint32_t &a, uint32_t &b) {
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "r"(smem_u32(p)));
}
RAT_DEVICE void st_global_v2(void *p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(a), "r"(b) : "memory");
}
RAT_DEVICE void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

}  // namespace rat
