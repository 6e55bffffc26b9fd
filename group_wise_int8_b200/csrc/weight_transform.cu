// Offline weight transform: U = G g G^T per (cout, cin) in fp64, rounded to
// fp32, then group-wise int8 over G consecutive input channels at fixed
// (tap, cout) ("Data-Free Group-Wise Fully Quantized Winograd Convolution via
// Learnable Scales": G = S_G V; Fig. 2, every stage group-wise quantised).
//
// One thread per (cout, cin); a CTA holds one quantisation group (G threads).
// The fp64 evaluation order is fixed: t[i][b] = fma-chain over a of
// G[i][a] g[a][b], U[i][j] = fma-chain over b of t[i][b] G[j][b], each chain
// ascending from +0.
#include "kernels.h"

namespace wino {
namespace {

template <int M>
__global__ void __launch_bounds__(256) weight_transform_kernel(WeightArgs wa, const float* __restrict__ w, int Cin,
                                                               int Cout, int G, int8_t* __restrict__ Uq,
                                                               float* __restrict__ sU) {
    constexpr int N = M + 2, N2 = N * N;
    __shared__ float red[8][64];
    __shared__ float scl[64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int ci = blockIdx.x * G + threadIdx.x;
    const int co = blockIdx.y;
    const int ng = Cin / G;

    double g[3][3];
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) g[a][b] = (double)w[(((size_t)co * 3 + a) * 3 + b) * Cin + ci];
    double t[N][3];
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int b = 0; b < 3; ++b) {
            double acc = 0.0;
#pragma unroll
            for (int a = 0; a < 3; ++a) acc = __fma_rn(wa.G[i * 3 + a], g[a][b], acc);
            t[i][b] = acc;
        }
    float u[64];
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) {
            double acc = 0.0;
#pragma unroll
            for (int b = 0; b < 3; ++b) acc = __fma_rn(t[i][b], wa.G[j * 3 + b], acc);
            u[i * N + j] = __double2float_rn(acc);
        }
    float a[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) a[k] = k < N2 ? fabsf(u[k]) : 0.0f;
    warp_max_scatter64(a, lane);
    red[warp][2 * lane] = a[0];
    red[warp][2 * lane + 1] = a[1];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int tap = 2 * lane + e;
            float amax = 0.0f;
            for (int i = 0; i < nwarps; ++i) amax = fmaxf(amax, red[i][tap]);
            const float s = group_scale(amax);
            scl[tap] = s;
            if (tap < N2) sU[((size_t)tap * ng + blockIdx.x) * Cout + co] = s;
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < N2; ++k) Uq[((size_t)k * Cout + co) * Cin + ci] = (int8_t)quant_code(u[k], scl[k]);
}

}  // namespace

cudaError_t launch_weight_transform(const WeightArgs& wa, int m, const float* w, int Cin, int Cout, int G,
                                    int8_t* Uq, float* sU, cudaStream_t st) {
    dim3 grid(Cin / G, Cout);
    if (m == 2)
        weight_transform_kernel<2><<<grid, G, 0, st>>>(wa, w, Cin, Cout, G, Uq, sU);
    else if (m == 4)
        weight_transform_kernel<4><<<grid, G, 0, st>>>(wa, w, Cin, Cout, G, Uq, sU);
    else
        weight_transform_kernel<6><<<grid, G, 0, st>>>(wa, w, Cin, Cout, G, Uq, sU);
    return cudaGetLastError();
}

}  // namespace wino
