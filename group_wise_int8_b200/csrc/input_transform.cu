// Input transform with group-wise int8 quantisation ("Data-Free Group-Wise
// Fully Quantized Winograd Convolution via Learnable Scales", Fig. 2: the
// input transform B^T d B is group-wise quantised).
//
// Tile t = (img*TH + ty)*TW + tx reads rows ty*m-1 .. ty*m+m and columns
// tx*m-1 .. tx*m+m of the NHWC input (zeros outside: stride 1, pad 1) and
// produces V = B^T d B per channel:
//   T1[i][l] = fma-chain over k of BT[i][k] d[k][l],
//   V[i][j]  = fma-chain over l of T1[i][l] BT[j][l]      (fp32, ascending, from +0;
//   exact-zero coefficients are skipped, which can change only the sign of a zero).
// Q then runs over G consecutive channels at fixed (tile, tap).
//
// CTA: TX consecutive tiles of one tile row x one quantisation group of G
// channels (128 threads, 256 for G = 256); one thread per (tile, channel),
// lanes along channels, so each warp-wide load of a pixel is contiguous.  The
// n x n patch is read straight from global memory (neighbouring tiles share
// two columns, which the L1 absorbs) and transformed in registers.  V then
// goes to shared memory (rows padded to 33 words), where lane l of the warp
// owns taps l and l + 32: it takes their absmax over the warp's 32 channels
// (the G/32 warps of a group combine theirs in shared memory), the group
// scale, and the 32 codes of each of its taps, packed into two 16-byte stores
// of the tap-major Vq.
#include "kernels.h"

namespace wino {
namespace {

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) {
    return __ldg(p);
}
template <>
__device__ __forceinline__ float load_as_float<uint16_t>(const uint16_t* p) {
    return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p)));
}

template <int M>
struct InCfg {
    static constexpr int N = M + 2, N2 = N * N;
    static constexpr int kPitch = 33;  // words per V row in shared memory
};

template <int M, uint64_t MASK, typename Tin, int G, int TX>
__global__ void __launch_bounds__(G* TX) input_transform_kernel(InputArgs p, TransformArgs tf) {
    constexpr int N = M + 2, N2 = N * N;
    constexpr int WPT = G / 32;      // warps per tile (= per group)
    constexpr int NW = TX * WPT;     // warps per CTA
    constexpr int P = InCfg<M>::kPitch;
    extern __shared__ float vbuf[];  // [NW][N2][P]
    __shared__ float red[NW][64];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row_id = blockIdx.y;  // img * TH + ty
    const int img = row_id / p.TH, ty = row_id - img * p.TH;
    const int tl = warp / WPT;
    const int tx = blockIdx.x * TX + tl;
    const bool valid = tx < p.TW;
    const int g = blockIdx.z;
    const int cw = g * G + (warp % WPT) * 32;  // first channel of this warp
    const long t = (long)row_id * p.TW + tx;
    const Tin* x = reinterpret_cast<const Tin*>(p.x);

    if (blockIdx.x == 0 && blockIdx.y == 0 && g == 0 && tid == 0) *p.err = 0;
    if (g == 0)
        for (int i = tid; i < TX * p.ngo; i += blockDim.x) {
            const int tt = i / p.ngo, k = i - tt * p.ngo;
            if (blockIdx.x * TX + tt < p.TW) p.amax[((size_t)row_id * p.TW + blockIdx.x * TX + tt) * p.ngo + k] = 0u;
        }

    {
        // 1. the n x n patch of channel cw + lane (zeros outside the image)
        float v[N][N];
#pragma unroll
        for (int r = 0; r < N; ++r) {
            const int yy = ty * M - 1 + r;
            const bool row_in = valid && yy >= 0 && yy < p.H;
            const Tin* xr = x + ((size_t)img * p.H + (row_in ? yy : 0)) * p.W * p.Cin + cw + lane;
#pragma unroll
            for (int l = 0; l < N; ++l) {
                const int xx = tx * M - 1 + l;
                v[r][l] = (row_in && xx >= 0 && xx < p.W) ? load_as_float<Tin>(xr + (size_t)xx * p.Cin) : 0.0f;
            }
        }
        // 2. V = B^T d B
#pragma unroll
        for (int l = 0; l < N; ++l) {
            float tcol[N];
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < N; ++k)
                    if ((MASK >> (i * N + k)) & 1ull) acc = __fmaf_rn(tf.BT[i * N + k], v[k][l], acc);
                tcol[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < N; ++i) v[i][l] = tcol[i];
        }
        float* vw = vbuf + (size_t)warp * N2 * P;
#pragma unroll
        for (int i = 0; i < N; ++i) {
#pragma unroll
            for (int j = 0; j < N; ++j) {
                float acc = 0.0f;
#pragma unroll
                for (int l = 0; l < N; ++l)
                    if ((MASK >> (j * N + l)) & 1ull) acc = __fmaf_rn(v[i][l], tf.BT[j * N + l], acc);
                vw[(i * N + j) * P + lane] = acc;   // 3. V row of tap (i, j), this lane's channel
            }
        }
    }
    __syncwarp();

    // 4. absmax of this lane's taps over the warp's 32 channels
    const float* vw = vbuf + (size_t)warp * N2 * P;
    float am[2] = {0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int tap = lane + 32 * e;
        if (tap < N2) {
            float a = 0.0f;
#pragma unroll 8
            for (int j = 0; j < 32; ++j) a = fmaxf(a, fabsf(vw[tap * P + j]));
            am[e] = a;
        }
    }
    if (WPT > 1) {
        red[warp][lane] = am[0];
        red[warp][lane + 32] = am[1];
        __syncthreads();
        const int leader = warp - warp % WPT;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < WPT; ++i) a = fmaxf(a, red[leader + i][lane + 32 * e]);
            am[e] = a;
        }
    }

    // 5. scales and codes of this lane's taps
    if (valid) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int tap = lane + 32 * e;
            if (tap >= N2) continue;
            const QScale q = make_qscale(am[e]);
            if (warp % WPT == 0) p.sV[((size_t)tap * (p.Cin / G) + g) * p.T_pad + t] = q.s;
            uint32_t w[8];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                uint32_t pk = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    pk |= ((uint32_t)(quant_code_fast(vw[tap * P + 4 * j4 + b], q) & 0xff)) << (8 * b);
                w[j4] = pk;
            }
            uint4* dst = reinterpret_cast<uint4*>(p.Vq + ((size_t)tap * p.T_pad + t) * p.Cin + cw);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

template <int M, uint64_t MASK, typename Tin, int G>
cudaError_t launch_g(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    constexpr int TX = G >= 128 ? 1 : 128 / G;
    constexpr int NW = TX * G / 32;
    const size_t smem = sizeof(float) * NW * InCfg<M>::N2 * InCfg<M>::kPitch;
    auto kern = input_transform_kernel<M, MASK, Tin, G, TX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.TW + TX - 1) / TX, a.N * a.TH, a.Cin / G);
    kern<<<grid, G * TX, smem, st>>>(a, tf);
    return cudaGetLastError();
}

template <int M, uint64_t MASK, typename Tin>
cudaError_t launch_cc(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    if (a.G == 32) return launch_g<M, MASK, Tin, 32>(a, tf, st);
    if (a.G == 64) return launch_g<M, MASK, Tin, 64>(a, tf, st);
    if (a.G == 256) return launch_g<M, MASK, Tin, 256>(a, tf, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_input_transform(const InputArgs& a, const TransformArgs& tf, int m, bool masked, bool bf16_in,
                                   cudaStream_t st) {
    if (m == 4) {
        if (bf16_in)
            return masked ? launch_cc<4, kMaskBT_F4, uint16_t>(a, tf, st) : launch_cc<4, kMaskAll, uint16_t>(a, tf, st);
        return masked ? launch_cc<4, kMaskBT_F4, float>(a, tf, st) : launch_cc<4, kMaskAll, float>(a, tf, st);
    }
    if (bf16_in)
        return masked ? launch_cc<6, kMaskBT_F6, uint16_t>(a, tf, st) : launch_cc<6, kMaskAll, uint16_t>(a, tf, st);
    return masked ? launch_cc<6, kMaskBT_F6, float>(a, tf, st) : launch_cc<6, kMaskAll, float>(a, tf, st);
}

}  // namespace wino
