// Shared device code of the Winograd library: the int8 quantiser, the warp
// absmax reduction and the kernel-parameter structs.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "plan.h"

namespace wino {

// Zero patterns (bit i*n+k) of the unscaled transforms for the standard
// point orders 0,1,-1,inf (F(2,3)), 0,1,-1,2,-2,inf (F(4,3)) and
// 0,1,-1,2,-2,1/2,-1/2,inf (F(6,3)).
// Diagonal scales keep the pattern.  The host verifies a plan's exact pattern
// is contained in the mask before choosing a masked kernel; otherwise the
// all-ones (generic) kernel runs.
constexpr uint64_t kMaskBT_F2 = 0x000000000000a665ull;
constexpr uint64_t kMaskAT_F2 = 0x00000000000000e7ull;
constexpr uint64_t kMaskBT_F4 = 0x0000000a9e79e795ull;
constexpr uint64_t kMaskAT_F4 = 0x0000000000f9e79full;
constexpr uint64_t kMaskBT_F6 = 0xaa7e7e7e7e7e7e55ull;
constexpr uint64_t kMaskAT_F6 = 0x0000fe7e7e7e7e7full;
constexpr uint64_t kMaskAll = ~0ull;

// The fp32 transforms as kernel arguments (they live in the constant bank),
// also as packed pairs (c, c) for the two-lane fp32 instructions.
struct TransformArgs {
    float BT[kMaxN * kMaxN];
    float AT[6 * kMaxN];
    uint64_t BTd[kMaxN * kMaxN];
    uint64_t ATd[6 * kMaxN];
};

struct WeightArgs {
    double G[kMaxN * 3];
};

// 1.5 * 2^23: adding it to |v| < 2^22 rounds v to the nearest integer (ties
// to even) and leaves that integer in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;
constexpr int kRoundMagicBits = 0x4B400000;

// Q for one value given the group scale s = absmax / 127 (fp32, IEEE):
// q = clamp(rne(v / s), -127, 127), q = 0 when s == 0.
__device__ __forceinline__ int quant_code(float v, float s) {
    if (s == 0.0f) return 0;
    const float r = __fdiv_rn(v, s);
    int q = __float_as_int(__fadd_rn(r, kRoundMagic)) - kRoundMagicBits;
    q = q > 127 ? 127 : q;
    q = q < -127 ? -127 : q;
    return q;
}

// Group scale from an absmax.
__device__ __forceinline__ float group_scale(float amax) { return __fdiv_rn(amax, 127.0f); }

// Packed fp32 pairs (sm_100): each lane of the pair is rounded exactly as the
// scalar instruction would round it.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// A group scale with its reciprocals for the quantisers below.
struct QScale {
    float s;
    float r;    // RN24(1 / s); 0 when s == 0 or s lies outside [2^-100, 2^100]
    double rd;  // RN53(1 / s); 0 when s == 0
};

__device__ __forceinline__ QScale make_qscale(float amax) {
    QScale q;
    q.s = group_scale(amax);
    q.r = (q.s >= 0x1p-100f && q.s <= 0x1p100f) ? __frcp_rn(q.s) : 0.0f;
    q.rd = q.s != 0.0f ? __drcp_rn((double)q.s) : 0.0;
    return q;
}

// max(a, |b|, |c|) in one three-input max (exact, like any max).
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

// The same code as quant_code(v, s) without a division or a branch.
// RN24(v/s) = (float)((double)v * RN53(1/s)) for fp32 v and s > 0: the exact
// quotient of two 24-bit numbers is never an fp32 rounding midpoint and lies at
// least 2^-49 (relative) away from every midpoint (write v - s*mid as a
// multiple of the lowest set bit of s*mid), while the fp64 product carries a
// relative error below 2^-51 (one rounding in the reciprocal, one in the
// product), so both round to the same fp32 value -- the argument by which
// double rounding through 53 bits is innocuous for a 24-bit quotient.  The
// integer step and the clamp then match quant_code exactly.
__device__ __forceinline__ int quant_code_fast(float v, QScale q) {
    const float r = __double2float_rn(__dmul_rn((double)v, q.rd));   // RN24(v / s); 0 when s == 0
    int c = __float_as_int(__fadd_rn(r, kRoundMagic)) - kRoundMagicBits;
    c = c > 127 ? 127 : c;
    return c < -127 ? -127 : c;
}

// Codes of four values of one group (|v| <= the group's absmax), in fp32
// pairs: t = RN(v * RN(1/s)) lies within 2.3e-5 of RN(v/s) (|v/s| < 127.0001;
// one rounding each in 1/s, in t and in RN(v/s), at most 2^-24 relative), so
// when every t is more than 2^-12 from a half-integer, rne(t) = rne(RN(v/s))
// and the clamp cannot act (|rne| <= 127).  a = t + 1.5*2^23 holds rne(t) in
// its low mantissa bits, so byte 0 of a's bits is the int8 code and k = a -
// 1.5*2^23 is rne(t) as a float.  Otherwise (about one value in 4000, or a
// scale outside [2^-100, 2^100]) the fp64 quotient decides.
struct Quad {
    uint64_t k01, k23;  // rne codes as floats
    uint32_t packed;    // the four int8 codes, value 0 in byte 0
};

__device__ __forceinline__ Quad quant4(float v0, float v1, float v2, float v3, const QScale& q) {
    Quad o;
    const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
    if (q.r != 0.0f || q.s == 0.0f) {
        const uint64_t r2 = f2_pack(q.r, q.r);
        const uint64_t t01 = f2_mul(f2_pack(v0, v1), r2), t23 = f2_mul(f2_pack(v2, v3), r2);
        const uint64_t a01 = f2_add(t01, magic2), a23 = f2_add(t23, magic2);
        o.k01 = f2_sub(a01, magic2);
        o.k23 = f2_sub(a23, magic2);
        float d0, d1, d2, d3;
        f2_unpack(f2_sub(t01, o.k01), d0, d1);
        f2_unpack(f2_sub(t23, o.k23), d2, d3);
        const float dmax = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fmaxf(fabsf(d2), fabsf(d3)));
        if (dmax < 0.5f - 0x1p-12f) {
            float a0, a1, a2, a3;
            f2_unpack(a01, a0, a1);
            f2_unpack(a23, a2, a3);
            o.packed = __byte_perm(__byte_perm(__float_as_uint(a0), __float_as_uint(a1), 0x0040),
                                   __byte_perm(__float_as_uint(a2), __float_as_uint(a3), 0x0040), 0x5410);
            return o;
        }
    }
    const int c0 = quant_code_fast(v0, q), c1 = quant_code_fast(v1, q);
    const int c2 = quant_code_fast(v2, q), c3 = quant_code_fast(v3, q);
    o.k01 = f2_pack((float)c0, (float)c1);
    o.k23 = f2_pack((float)c2, (float)c3);
    o.packed = (uint32_t)(c0 & 0xff) | ((uint32_t)(c1 & 0xff) << 8) | ((uint32_t)(c2 & 0xff) << 16) |
               ((uint32_t)(c3 & 0xff) << 24);
    return o;
}

// Codes of NV values of one group (NV a multiple of 4), packed four per word,
// by the argument of quant4 with a single check for all NV values (the
// fallback, taken when any of them lies near a half-integer, is quant_code_fast
// for all of them).
template <int NV>
__device__ __forceinline__ void quant_chunk(const float (&v)[NV], const QScale& q, uint32_t (&w)[NV / 4]) {
    const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
    if (q.r != 0.0f || q.s == 0.0f) {
        const uint64_t r2 = f2_pack(q.r, q.r);
        uint64_t a[NV / 2];
        float dmax = 0.0f;
#pragma unroll
        for (int i = 0; i < NV / 2; ++i) {
            const uint64_t t = f2_mul(f2_pack(v[2 * i], v[2 * i + 1]), r2);
            a[i] = f2_add(t, magic2);
            float d0, d1;
            f2_unpack(f2_sub(t, f2_sub(a[i], magic2)), d0, d1);
            dmax = max_abs3(dmax, d0, d1);
        }
        if (dmax < 0.5f - 0x1p-12f) {
#pragma unroll
            for (int i = 0; i < NV / 4; ++i) {
                float a0, a1, a2, a3;
                f2_unpack(a[2 * i], a0, a1);
                f2_unpack(a[2 * i + 1], a2, a3);
                w[i] = __byte_perm(__byte_perm(__float_as_uint(a0), __float_as_uint(a1), 0x0040),
                                   __byte_perm(__float_as_uint(a2), __float_as_uint(a3), 0x0040), 0x5410);
            }
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < NV / 4; ++i) {
        const int c0 = quant_code_fast(v[4 * i], q), c1 = quant_code_fast(v[4 * i + 1], q);
        const int c2 = quant_code_fast(v[4 * i + 2], q), c3 = quant_code_fast(v[4 * i + 3], q);
        w[i] = (uint32_t)(c0 & 0xff) | ((uint32_t)(c1 & 0xff) << 8) | ((uint32_t)(c2 & 0xff) << 16) |
               ((uint32_t)(c3 & 0xff) << 24);
    }
}

// Recursive-halving max over the 32 lanes of a warp for 64 values per lane.
// a[0..63] holds this lane's values; on return a[0], a[1] hold the maxima
// over all lanes of entries 2*lane and 2*lane + 1.
__device__ __forceinline__ void warp_max_scatter64(float (&a)[64], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int h = 32 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? a[i] : a[i + h];
            const float keep = upper ? a[i + h] : a[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            a[i] = fmaxf(keep, recv);
        }
    }
}

// Index checks of the debug build (compiled with -DWINO_DEBUG): an access whose
// element index i lies outside its buffer of n elements is skipped and recorded
// in the device error word as kDevErrBounds (first error wins); nothing traps.
// In the release build every check is the constant true and costs nothing.
constexpr int kDevErrBounds = 2;
#ifdef WINO_DEBUG
__device__ __forceinline__ bool in_bounds(size_t i, size_t n, int* err) {
    if (i < n) return true;
    if (err) atomicCAS(err, 0, kDevErrBounds);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(size_t, size_t, int*) { return true; }
#endif

}  // namespace wino
