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
// CTA: TX consecutive tiles of one tile row x CC channels; one thread per
// (tile, channel), lanes along channels.  The halo patch is staged in shared
// memory with 16-byte loads; the per-(tile, tap) absmax of a 32-channel warp
// is a recursive-halving shuffle reduction (each lane ends with two taps),
// combined across the G/32 warps of a group in shared memory; the int8 codes
// are staged in shared memory and written with 16-byte stores.
#include "kernels.h"

namespace wino {
namespace {

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) {
    return *p;
}
template <>
__device__ __forceinline__ float load_as_float<uint16_t>(const uint16_t* p) {
    return bf16_bits_to_float(*p);
}

template <int M, uint64_t MASK, typename Tin, int CC, int TX>
__global__ void __launch_bounds__(CC* TX) input_transform_kernel(InputArgs p, TransformArgs tf) {
    constexpr int N = M + 2, N2 = N * N, PW = TX * M + 2;
    constexpr int VEC = 16 / sizeof(Tin);
    constexpr int WPT = CC / 32;  // warps per tile
    extern __shared__ __align__(16) unsigned char smem[];
    Tin* patch = reinterpret_cast<Tin*>(smem);                                 // [N][PW][CC]
    float* red = reinterpret_cast<float*>(smem + sizeof(Tin) * N * PW * CC);   // [TX*WPT][64]
    float* scl = red + TX * WPT * 64;                                          // [TX*WPT][64] (per group leader)
    int8_t* outb = reinterpret_cast<int8_t*>(scl + TX * WPT * 64);             // [TX][N2][CC]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row_id = blockIdx.y;  // img * TH + ty
    const int img = row_id / p.TH, ty = row_id - img * p.TH;
    const int tx0 = blockIdx.x * TX;
    const int c0 = blockIdx.z * CC;
    const Tin* x = reinterpret_cast<const Tin*>(p.x);

    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && tid == 0) *p.err = 0;
    if (blockIdx.z == 0) {
        for (int i = tid; i < TX * p.ngo; i += blockDim.x) {
            const int tl = i / p.ngo, k = i - tl * p.ngo;
            if (tx0 + tl < p.TW) p.amax[((size_t)row_id * p.TW + tx0 + tl) * p.ngo + k] = 0u;
        }
    }

    // 1. halo patch -> shared memory (zeros outside the image)
    for (int v = tid; v < N * PW * (CC / VEC); v += blockDim.x) {
        const int cv = v % (CC / VEC);
        const int rest = v / (CC / VEC);
        const int col = rest % PW, r = rest / PW;
        const int yy = ty * M - 1 + r, xx = tx0 * M - 1 + col;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (yy >= 0 && yy < p.H && xx >= 0 && xx < p.W)
            val = *reinterpret_cast<const uint4*>(x + (((size_t)img * p.H + yy) * p.W + xx) * p.Cin + c0 + cv * VEC);
        *reinterpret_cast<uint4*>(patch + ((size_t)(r * PW + col) * CC + cv * VEC)) = val;
    }
    __syncthreads();

    // 2. transform for (tile tl, channel cl)
    const int tl = warp / WPT;
    const int cl = (warp % WPT) * 32 + lane;
    float v[N][N];
#pragma unroll
    for (int r = 0; r < N; ++r)
#pragma unroll
        for (int l = 0; l < N; ++l) v[r][l] = load_as_float<Tin>(patch + (size_t)(r * PW + tl * M + l) * CC + cl);
#pragma unroll
    for (int l = 0; l < N; ++l) {
        float t[N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < N; ++k)
                if ((MASK >> (i * N + k)) & 1ull) acc = __fmaf_rn(tf.BT[i * N + k], v[k][l], acc);
            t[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) v[i][l] = t[i];
    }
#pragma unroll
    for (int i = 0; i < N; ++i) {
        float t[N];
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float acc = 0.0f;
#pragma unroll
            for (int l = 0; l < N; ++l)
                if ((MASK >> (j * N + l)) & 1ull) acc = __fmaf_rn(v[i][l], tf.BT[j * N + l], acc);
            t[j] = acc;
        }
#pragma unroll
        for (int j = 0; j < N; ++j) v[i][j] = t[j];
    }

    // 3. per-(tile, tap) absmax over this warp's 32 channels
    {
        float a[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) a[k] = k < N2 ? fabsf(v[k / N][k % N]) : 0.0f;
        warp_max_scatter64(a, lane);
        red[warp * 64 + 2 * lane] = a[0];
        red[warp * 64 + 2 * lane + 1] = a[1];
    }
    __syncthreads();

    // 4. group scales: the first warp of each group combines its G/32 warps
    const int wpg = p.G / 32;
    const int leader = warp - (warp % wpg);
    const int ng = p.Cin / p.G;
    const int tx = tx0 + tl;
    const long t = (long)row_id * p.TW + tx;
    if (warp == leader) {
        const int g = (c0 + (warp % WPT) * 32) / p.G;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int tap = 2 * lane + e;
            float amax = 0.0f;
            for (int i = 0; i < wpg; ++i) amax = fmaxf(amax, red[(warp + i) * 64 + tap]);
            const float s = group_scale(amax);
            scl[warp * 64 + tap] = s;
            if (tap < N2 && tx < p.TW) p.sV[((size_t)tap * ng + g) * p.T_pad + t] = s;
        }
    }
    __syncthreads();

    // 5. int8 codes -> shared staging
#pragma unroll
    for (int k = 0; k < N2; ++k)
        outb[(tl * N2 + k) * CC + cl] = (int8_t)quant_code(v[k / N][k % N], scl[leader * 64 + k]);
    __syncthreads();

    // 6. 16-byte stores of Vq[t][tap][c0 .. c0+CC)
    for (int i = tid; i < TX * N2 * (CC / 16); i += blockDim.x) {
        const int cv = i % (CC / 16);
        const int rest = i / (CC / 16);
        const int tap = rest % N2, tl2 = rest / N2;
        if (tx0 + tl2 >= p.TW) continue;
        const size_t t2 = (size_t)row_id * p.TW + tx0 + tl2;
        *reinterpret_cast<uint4*>(p.Vq + (t2 * N2 + tap) * p.Cin + c0 + cv * 16) =
            *reinterpret_cast<const uint4*>(outb + (tl2 * N2 + tap) * CC + cv * 16);
    }
}

template <int M, uint64_t MASK, typename Tin, int CC, int TX>
cudaError_t launch_one(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    constexpr int N = M + 2, N2 = N * N, PW = TX * M + 2, WPT = CC / 32;
    const size_t smem = sizeof(Tin) * N * PW * CC + 2 * sizeof(float) * TX * WPT * 64 + (size_t)TX * N2 * CC;
    auto kern = input_transform_kernel<M, MASK, Tin, CC, TX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.TW + TX - 1) / TX, a.N * a.TH, a.Cin / CC);
    kern<<<grid, CC * TX, smem, st>>>(a, tf);
    return cudaGetLastError();
}

template <int M, uint64_t MASK, typename Tin>
cudaError_t launch_cc(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    // channel chunk: a multiple of G dividing Cin; 256 threads per CTA
    if (a.G == 256) return launch_one<M, MASK, Tin, 256, 1>(a, tf, st);
    if (a.Cin % 64 == 0) return launch_one<M, MASK, Tin, 64, 4>(a, tf, st);
    if (a.G == 32) return launch_one<M, MASK, Tin, 32, 8>(a, tf, st);
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
