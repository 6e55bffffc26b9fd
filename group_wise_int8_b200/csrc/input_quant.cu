// Group-wise int8 on the layer input itself (alternative reading of where the
// input side is quantised; "Data-Free Group-Wise Fully Quantized Winograd
// Convolution via Learnable Scales", Eqs. (14)-(16), where the input transform
// carries a scale of x besides the two of B).
//
// x [N][H][W][Cin] is viewed as a flat run of groups of G consecutive channels of
// one pixel (Cin % G == 0, so a group never crosses a pixel).  Each group gets
// s = absmax / 127 and every value becomes s * clamp(rne(x / s), +-127) in fp32;
// the input transform then reads these fp32 values.
//
// Each lane owns 8 consecutive values (one 16-byte bf16 load or two 16-byte fp32
// loads), so G / 8 lanes share a group and combine their absmax with xor
// shuffles; a warp covers 256 values per step of its grid-stride loop.  The codes
// come from the division-free exact quantiser (quant4) and s * q is one fp32
// multiply per value.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace wino {
namespace {

template <typename Tin>
__device__ __forceinline__ void load8(const Tin* p, float* v);
template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* p, float* v) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* v) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename Tin, int G>
__global__ void __launch_bounds__(256) input_quant_kernel(const Tin* __restrict__ x, long elems,
                                                          float* __restrict__ xq) {
    grid_dependents_launch();
    grid_dependency_wait();
    constexpr int kLanes = G / 8;  // lanes per group: 4, 8 or 32
    const int lane = threadIdx.x & 31;
    const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long nwarps = ((long)gridDim.x * blockDim.x) >> 5;
    for (long base = warp * 256; base < elems; base += nwarps * 256) {
        const long e = base + 8 * lane;
        // elems is a multiple of G (and G of 8): a group, hence a lane's 8 values, lies wholly in
        // range or wholly out; lanes past the end take part in the shuffles with zeros
        const bool live = e < elems && in_bounds(e + 7, elems, nullptr);
        float v[8];
        if (live) {
            load8<Tin>(x + e, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
        for (int off = 1; off < kLanes; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        // codes without a division (quant4: exact, with its own fallback), then s * q in fp32
        const QScale q = make_qscale(amax);
        const uint64_t s2 = f2_pack(q.s, q.s);
        const Quad a = quant4(v[0], v[1], v[2], v[3], q), b = quant4(v[4], v[5], v[6], v[7], q);
        if (live) {
            ulonglong2* dst = reinterpret_cast<ulonglong2*>(xq + e);
            dst[0] = make_ulonglong2(f2_mul(s2, a.k01), f2_mul(s2, a.k23));
            dst[1] = make_ulonglong2(f2_mul(s2, b.k01), f2_mul(s2, b.k23));
        }
    }
}

template <typename Tin>
cudaError_t launch_t(const void* x, long elems, int G, float* xq, int num_sms, cudaStream_t st) {
    const long warps = (elems + 255) / 256;
    const long blocks = std::min<long>((warps + 7) / 8, (long)num_sms * 8);
    const dim3 grid((unsigned)std::max<long>(blocks, 1)), block(256);
    const Tin* xp = static_cast<const Tin*>(x);
    if (G == 32) return launch_dependent(input_quant_kernel<Tin, 32>, grid, block, 0, st, xp, elems, xq);
    if (G == 64) return launch_dependent(input_quant_kernel<Tin, 64>, grid, block, 0, st, xp, elems, xq);
    if (G == 256) return launch_dependent(input_quant_kernel<Tin, 256>, grid, block, 0, st, xp, elems, xq);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_input_quant(const void* x, bool bf16_in, long elems, int G, float* xq, int num_sms,
                               cudaStream_t st) {
    if (elems % 8 != 0 || elems % G != 0) return cudaErrorInvalidValue;
    return bf16_in ? launch_t<uint16_t>(x, elems, G, xq, num_sms, st) : launch_t<float>(x, elems, G, xq, num_sms, st);
}

}  // namespace wino
