// Output transform of the group-wise fully quantized Winograd convolution
// ("Data-Free Group-Wise Fully Quantized Winograd Convolution via Learnable
// Scales": A^T = V^T S_A; Fig. 2, the output transform's input Y is
// group-wise quantised; "Core claim": Y's cross-shaped per-tap spread).
//
// Per (tile, cout): sY = absmax/127 of the (tile, G-cout) group over all n*n
// taps; Yd = sY * Yq (fp32); Z[i][nu] = fma-chain over xi of AT[i][xi] Yd[xi][nu];
// o[i][j] = fma-chain over nu of Z[i][nu] AT[j][nu]; cropped to the image and
// written NHWC in fp32 or bf16 (round to nearest even).
// The Y source is either the int8 Yq the GEMM's quantising pass wrote, or the
// fp32 Y of the single-pass GEMM, requantised here with the same Q.
// One thread per (tile, pair of adjacent couts): the pair shares its Y group,
// so every step runs on packed fp32 pairs (one two-lane instruction per pair,
// the per-cout chains and their order unchanged).  Lanes run along cout
// pairs: every tap load and output store of a warp is contiguous.  Z is built
// one column of Y at a time, so only Z and one Y column are live.
#include "kernels.h"

namespace wino {
namespace {

// int8 codes (bytes 0 and 1 of x) to exact fp32 values without a conversion
// instruction: byte ^ 0x80 placed in the low mantissa of 1.5*2^23 is
// 1.5*2^23 + 128 + q.
__device__ __forceinline__ uint64_t codes2_to_f2(uint32_t x) {
    const uint32_t b = x ^ 0x8080u;
    const uint32_t lo = __byte_perm(b, 0x4B400000u, 0x7640);
    const uint32_t hi = __byte_perm(b, 0x4B400000u, 0x7641);
    const float off = kRoundMagic + 128.0f;
    return f2_sub(f2_pack(__uint_as_float(lo), __uint_as_float(hi)), f2_pack(off, off));
}

template <int M, uint64_t MASK, bool SRC_Y32, bool BF16_OUT, bool DEBUG>
__global__ void __launch_bounds__(128, 4) output_transform_kernel(OutputArgs p, TransformArgs tf) {
    constexpr int N = M + 2;
    grid_dependents_launch();
    grid_dependency_wait();
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const int cpairs = p.Cout >> 1;
    const long t = i / cpairs;
    const int co = 2 * (int)(i - t * cpairs);
    if (t >= p.T) return;
    const int cg = co / p.G;
    const QScale qs = make_qscale(__uint_as_float(p.amax[(size_t)t * p.ngo + cg]));
    if (DEBUG && co % p.G == 0) p.sY_dbg[(size_t)t * p.ngo + cg] = qs.s;
    const uint64_t s2 = f2_pack(qs.s, qs.s);

    const size_t base = (size_t)t * p.Cout + co;   // Yq / Y32 are tap-major [n2][T][Cout]
    const size_t tstride = (size_t)p.T * p.Cout;
    uint64_t Z[M][N];                              // (co, co + 1) pairs
#pragma unroll
    for (int nu = 0; nu < N; ++nu) {
        uint64_t Yc[N];                            // column nu of Yd: taps xi * N + nu
        if (SRC_Y32) {
#pragma unroll
            for (int xi = 0; xi < N; xi += 2) {
                const float2 a = *reinterpret_cast<const float2*>(p.Y32 + base + (size_t)(xi * N + nu) * tstride);
                const float2 b = *reinterpret_cast<const float2*>(p.Y32 + base + (size_t)((xi + 1) * N + nu) * tstride);
                const Quad qd = quant4(a.x, a.y, b.x, b.y, qs);
                Yc[xi] = f2_mul(s2, qd.k01);
                Yc[xi + 1] = f2_mul(s2, qd.k23);
                if (DEBUG) {
                    *reinterpret_cast<uint16_t*>(p.Yq_dbg + base + (size_t)(xi * N + nu) * tstride) =
                        (uint16_t)(qd.packed & 0xffffu);
                    *reinterpret_cast<uint16_t*>(p.Yq_dbg + base + (size_t)((xi + 1) * N + nu) * tstride) =
                        (uint16_t)(qd.packed >> 16);
                }
            }
        } else {
#pragma unroll
            for (int xi = 0; xi < N; ++xi) {
                const uint32_t x = *reinterpret_cast<const uint16_t*>(p.Yq + base + (size_t)(xi * N + nu) * tstride);
                Yc[xi] = f2_mul(s2, codes2_to_f2(x));
            }
        }
#pragma unroll
        for (int r = 0; r < M; ++r) {
            uint64_t acc = 0ull;
#pragma unroll
            for (int xi = 0; xi < N; ++xi)
                if ((MASK >> (r * N + xi)) & 1ull) acc = f2_fma(tf.ATd[r * N + xi], Yc[xi], acc);
            Z[r][nu] = acc;
        }
    }
    const int TT = p.TH * p.TW;
    const int img = (int)(t / TT);
    const int rem = (int)(t - (long)img * TT);
    const int ty = rem / p.TW, tx = rem - ty * p.TW;
#pragma unroll
    for (int r = 0; r < M; ++r) {
        const int yy = ty * M + r;
        if (yy >= p.H) break;
#pragma unroll
        for (int c = 0; c < M; ++c) {
            const int xx = tx * M + c;
            if (xx >= p.W) break;
            uint64_t acc = 0ull;
#pragma unroll
            for (int nu = 0; nu < N; ++nu)
                if ((MASK >> (c * N + nu)) & 1ull) acc = f2_fma(Z[r][nu], tf.ATd[c * N + nu], acc);
            float o0, o1;
            f2_unpack(acc, o0, o1);
            const size_t o = (((size_t)img * p.H + yy) * p.W + xx) * p.Cout + co;
            if (BF16_OUT)
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p.out) + o) =
                    __floats2bfloat162_rn(o0, o1);
            else
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + o) = make_float2(o0, o1);
        }
    }
}

template <int M, uint64_t MASK>
cudaError_t launch_m(const OutputArgs& a, const TransformArgs& tf, bool src_y32, bool bf16_out, bool debug,
                     cudaStream_t st) {
    const long threads = a.T * (long)(a.Cout / 2);
    const dim3 grid((unsigned)((threads + 127) / 128));
#define WINO_OUT_LAUNCH(Y32, BF, DBG) \
    return launch_dependent(output_transform_kernel<M, MASK, Y32, BF, DBG>, grid, dim3(128), 0, st, a, tf)
    if (src_y32) {
        if (bf16_out) {
            if (debug) WINO_OUT_LAUNCH(true, true, true); else WINO_OUT_LAUNCH(true, true, false);
        } else {
            if (debug) WINO_OUT_LAUNCH(true, false, true); else WINO_OUT_LAUNCH(true, false, false);
        }
    } else {
        if (bf16_out) {
            if (debug) WINO_OUT_LAUNCH(false, true, true); else WINO_OUT_LAUNCH(false, true, false);
        } else {
            if (debug) WINO_OUT_LAUNCH(false, false, true); else WINO_OUT_LAUNCH(false, false, false);
        }
    }
#undef WINO_OUT_LAUNCH
    return cudaErrorInvalidValue;  // not reached
}

}  // namespace

cudaError_t launch_output_transform(const OutputArgs& a, const TransformArgs& tf, int m, bool masked, bool src_y32,
                                    bool bf16_out, cudaStream_t st) {
    const bool debug = a.sY_dbg != nullptr;
    if (m == 2)
        return masked ? launch_m<2, kMaskAT_F2>(a, tf, src_y32, bf16_out, debug, st)
                      : launch_m<2, kMaskAll>(a, tf, src_y32, bf16_out, debug, st);
    if (m == 4)
        return masked ? launch_m<4, kMaskAT_F4>(a, tf, src_y32, bf16_out, debug, st)
                      : launch_m<4, kMaskAll>(a, tf, src_y32, bf16_out, debug, st);
    return masked ? launch_m<6, kMaskAT_F6>(a, tf, src_y32, bf16_out, debug, st)
                  : launch_m<6, kMaskAll>(a, tf, src_y32, bf16_out, debug, st);
}

}  // namespace wino
