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
// lanes along channels.  One 4-D TMA box brings the CTA's halo patch
// (n rows x TX*m+2 columns x G channels; outside the image the box reads
// zeros, which is the pad-1 border) into shared memory; each thread reads its
// n x n patch from there and transforms it in registers.  V then goes to
// shared memory (rows padded to 36 words: 16-byte reads without bank
// conflicts), where lane l of the warp owns taps l and l + 32: it takes their
// absmax over the warp's 32 channels (the G/32 warps of a group combine theirs
// in shared memory), the group scale, and the 32 codes of each of its taps
// (quant4), packed into two 16-byte stores of the tap-major Vq.
#include "kernels.h"
#include "sm100.cuh"

namespace wino {
namespace {

template <typename T>
__device__ __forceinline__ float to_float(T v);
template <>
__device__ __forceinline__ float to_float<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ float to_float<uint16_t>(uint16_t v) {
    return bf16_bits_to_float(v);
}

template <int M, typename Tin, int G, int TX>
struct InCfg {
    static constexpr int N = M + 2, N2 = N * N;
    static constexpr int kPitch = 36;                   // words per V row in shared memory
    static constexpr int kNW = TX * G / 32;             // warps per CTA
    static constexpr int kPW = TX * M + 2;              // patch columns
    static constexpr size_t kPatchBytes = sizeof(Tin) * N * kPW * G;
    static constexpr size_t kPatchOff = 0;
    static constexpr size_t kVbufOff = (kPatchBytes + 127) / 128 * 128;
    static constexpr size_t kSmem = kVbufOff + sizeof(float) * kNW * N2 * kPitch;
};

template <int M, uint64_t MASK, typename Tin, int G, int TX>
__global__ void __launch_bounds__(G* TX) input_transform_kernel(const __grid_constant__ CUtensorMap tmX, InputArgs p,
                                                                TransformArgs tf) {
    using Cfg = InCfg<M, Tin, G, TX>;
    constexpr int N = M + 2, N2 = N * N, P = Cfg::kPitch, PW = Cfg::kPW;
    constexpr int WPT = G / 32;      // warps per tile (= per group)
    extern __shared__ __align__(128) unsigned char smem[];
    const Tin* patch = reinterpret_cast<const Tin*>(smem + Cfg::kPatchOff);   // [N][PW][G]
    float* vbuf = reinterpret_cast<float*>(smem + Cfg::kVbufOff);            // [NW][N2][P]
    __shared__ float red[Cfg::kNW][64];
    __shared__ uint64_t bar;
    __shared__ int load_ok;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_dependents_launch();
    grid_dependency_wait();
    const int row_id = blockIdx.y;  // img * TH + ty
    const int img = row_id / p.TH, ty = row_id - img * p.TH;
    const int tl = warp / WPT;
    const int tx0 = blockIdx.x * TX;
    const int tx = tx0 + tl;
    const bool valid = tx < p.TW;
    const int g = blockIdx.z;
    const int cl = (warp % WPT) * 32;  // first channel of this warp within the group
    const int cw = g * G + cl;
    const long t = (long)row_id * p.TW + tx;

    if (tid == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        sm100::mbar_arrive_expect_tx(&bar, (uint32_t)Cfg::kPatchBytes);
        sm100::tma_load_4d(smem + Cfg::kPatchOff, &tmX, &bar, g * G, tx0 * M - 1, ty * M - 1, img);
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && g == 0 && tid == 0) *p.err = 0;
    if (g == 0)
        for (int i = tid; i < TX * p.ngo; i += blockDim.x) {
            const int tt = i / p.ngo, k = i - tt * p.ngo;
            if (tx0 + tt < p.TW) p.amax[((size_t)row_id * p.TW + tx0 + tt) * p.ngo + k] = 0u;
        }
    if (tid == 0) {
        load_ok = 1;
        const unsigned long long t0 = sm100::globaltimer();
        while (!sm100::mbar_try_wait(&bar, 0))
            if (sm100::globaltimer() - t0 > sm100::kWaitLimitNs) {
                load_ok = 0;
                atomicCAS(p.err, 0, sm100::kDevErrTimeout);
                break;
            }
    }
    __syncthreads();
    if (!load_ok) return;   // uniform across the CTA; the host reads the error word

    {
        // 1.-2. the n x n patch of channel cw + lane, V = B^T d B
        float v[N][N];
#pragma unroll
        for (int r = 0; r < N; ++r)
#pragma unroll
            for (int l = 0; l < N; ++l) v[r][l] = to_float<Tin>(patch[(r * PW + tl * M + l) * G + cl + lane]);
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
            const float4* row = reinterpret_cast<const float4*>(vw + tap * P);
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 q = row[j];
                a = fmaxf(a, fmaxf(fmaxf(fabsf(q.x), fabsf(q.y)), fmaxf(fabsf(q.z), fabsf(q.w))));
            }
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
            const float4* row = reinterpret_cast<const float4*>(vw + tap * P);
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 x4 = row[j];
                w[j] = quant4(x4.x, x4.y, x4.z, x4.w, q).packed;
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
    using Cfg = InCfg<M, Tin, G, TX>;
    // x [N][H][W][Cin] as a 4-D tensor (Cin, W, H, N); box G x (TX*m+2) x n x 1
    CUtensorMap tm;
    const cuuint64_t es = sizeof(Tin);
    const cuuint64_t dims[4] = {(cuuint64_t)a.Cin, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.N};
    const cuuint64_t strides[3] = {es * a.Cin, es * a.Cin * a.W, es * a.Cin * a.W * a.H};
    const cuuint32_t box[4] = {(cuuint32_t)G, (cuuint32_t)Cfg::kPW, (cuuint32_t)Cfg::N, 1u};
    if (!make_tensor_map(&tm, sizeof(Tin) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                         a.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = input_transform_kernel<M, MASK, Tin, G, TX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.TW + TX - 1) / TX, a.N * a.TH, a.Cin / G);
    return launch_dependent(kern, grid, dim3(G * TX), Cfg::kSmem, st, tm, a, tf);
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
