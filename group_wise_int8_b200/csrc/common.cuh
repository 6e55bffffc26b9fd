// Shared device code of the Winograd library: the int8 quantiser, the warp
// absmax reduction and the kernel-parameter structs.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "plan.h"

namespace wino {

// Zero patterns (bit i*n+k) of the unscaled transforms for the standard
// point orders 0,1,-1,2,-2,inf (F(4,3)) and 0,1,-1,2,-2,1/2,-1/2,inf (F(6,3)).
// Diagonal scales keep the pattern.  The host verifies a plan's exact pattern
// is contained in the mask before choosing a masked kernel; otherwise the
// all-ones (generic) kernel runs.
constexpr uint64_t kMaskBT_F4 = 0x0000000a9e79e795ull;
constexpr uint64_t kMaskAT_F4 = 0x0000000000f9e79full;
constexpr uint64_t kMaskBT_F6 = 0xaa7e7e7e7e7e7e55ull;
constexpr uint64_t kMaskAT_F6 = 0x0000fe7e7e7e7e7full;
constexpr uint64_t kMaskAll = ~0ull;

// The fp32 transforms as kernel arguments (they live in the constant bank).
struct TransformArgs {
    float BT[kMaxN * kMaxN];
    float AT[6 * kMaxN];
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

// A group scale with the fp64 reciprocal of its value, for quant_code_fast.
struct QScale {
    float s;
    double rd;  // RN53(1 / s); 0 when s == 0
};

__device__ __forceinline__ QScale make_qscale(float amax) {
    QScale q;
    q.s = group_scale(amax);
    q.rd = q.s != 0.0f ? __drcp_rn((double)q.s) : 0.0;
    return q;
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

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

}  // namespace wino
