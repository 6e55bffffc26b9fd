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
// One thread per (tile, cout); lanes along cout, so every tap load and every
// output store of a warp is contiguous.
#include "kernels.h"

namespace wino {
namespace {

template <int M, uint64_t MASK, bool SRC_Y32, bool BF16_OUT, bool DEBUG>
__global__ void __launch_bounds__(256) output_transform_kernel(OutputArgs p, TransformArgs tf) {
    constexpr int N = M + 2, N2 = N * N;
    grid_dependents_launch();
    grid_dependency_wait();
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long t = i / p.Cout;
    const int co = (int)(i - t * p.Cout);
    if (t >= p.T) return;
    const int cg = co / p.G;
    const QScale qs = make_qscale(__uint_as_float(p.amax[(size_t)t * p.ngo + cg]));
    const float s = qs.s;
    if (DEBUG && co % p.G == 0) p.sY_dbg[(size_t)t * p.ngo + cg] = s;

    float Y[N][N];
    const size_t base = (size_t)t * p.Cout + co;   // Yq / Y32 are tap-major [n2][T][Cout]
    const size_t tstride = (size_t)p.T * p.Cout;
    if (SRC_Y32) {
        const uint64_t s2 = f2_pack(s, s);
#pragma unroll
        for (int k = 0; k < N2; k += 4) {
            const float* src = p.Y32 + base + (size_t)k * tstride;
            const Quad qd = quant4(src[0], src[tstride], src[2 * tstride], src[3 * tstride], qs);
            f2_unpack(f2_mul(s2, qd.k01), Y[k / N][k % N], Y[(k + 1) / N][(k + 1) % N]);
            f2_unpack(f2_mul(s2, qd.k23), Y[(k + 2) / N][(k + 2) % N], Y[(k + 3) / N][(k + 3) % N]);
            if (DEBUG)
                for (int e = 0; e < 4; ++e) p.Yq_dbg[base + (size_t)(k + e) * tstride] = (int8_t)(qd.packed >> (8 * e));
        }
    } else {
#pragma unroll
        for (int k = 0; k < N2; ++k) Y[k / N][k % N] = __fmul_rn(s, (float)p.Yq[base + (size_t)k * tstride]);
    }
    float Z[M][N];
#pragma unroll
    for (int r = 0; r < M; ++r)
#pragma unroll
        for (int nu = 0; nu < N; ++nu) {
            float acc = 0.0f;
#pragma unroll
            for (int xi = 0; xi < N; ++xi)
                if ((MASK >> (r * N + xi)) & 1ull) acc = __fmaf_rn(tf.AT[r * N + xi], Y[xi][nu], acc);
            Z[r][nu] = acc;
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
            float acc = 0.0f;
#pragma unroll
            for (int nu = 0; nu < N; ++nu)
                if ((MASK >> (c * N + nu)) & 1ull) acc = __fmaf_rn(Z[r][nu], tf.AT[c * N + nu], acc);
            const size_t o = (((size_t)img * p.H + yy) * p.W + xx) * p.Cout + co;
            if (BF16_OUT)
                reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(acc);
            else
                reinterpret_cast<float*>(p.out)[o] = acc;
        }
    }
}

template <int M, uint64_t MASK>
cudaError_t launch_m(const OutputArgs& a, const TransformArgs& tf, bool src_y32, bool bf16_out, bool debug,
                     cudaStream_t st) {
    const long threads = a.T * (long)a.Cout;
    const dim3 grid((unsigned)((threads + 255) / 256));
#define WINO_OUT_LAUNCH(Y32, BF, DBG) \
    return launch_dependent(output_transform_kernel<M, MASK, Y32, BF, DBG>, grid, dim3(256), 0, st, a, tf)
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
    if (m == 4)
        return masked ? launch_m<4, kMaskAT_F4>(a, tf, src_y32, bf16_out, debug, st)
                      : launch_m<4, kMaskAll>(a, tf, src_y32, bf16_out, debug, st);
    return masked ? launch_m<6, kMaskAT_F6>(a, tf, src_y32, bf16_out, debug, st)
                  : launch_m<6, kMaskAll>(a, tf, src_y32, bf16_out, debug, st);
}

}  // namespace wino
