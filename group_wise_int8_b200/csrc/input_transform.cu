// Input transform with group-wise int8 quantisation ("Data-Free Group-Wise
// Fully Quantized Winograd Convolution via Learnable Scales", Fig. 2: the input
// transform B^T d B is group-wise quantised).
//
// Tile t = (img*TH + ty)*TW + tx reads rows ty*m-1 .. ty*m+m and columns
// tx*m-1 .. tx*m+m of the NHWC input (zeros outside: stride 1, pad 1) and
// produces V = B^T d B per channel:
//   T1[i][l] = fma-chain over k of BT[i][k] d[k][l],
//   V[i][j]  = fma-chain over l of T1[i][l] BT[j][l]      (fp32, ascending, from +0;
//   exact-zero coefficients are skipped, which can change only the sign of a zero).
// Q then runs over G consecutive channels at fixed (tile, tap).
//
// CTA: TX consecutive tiles of one tile row (TX = TW, or a balanced share of
// a long row) and one quantisation group of G channels; each thread owns one
// tile and a pair of adjacent channels, so both chains run as one two-lane
// fp32 instruction per step (the per-channel chains are unchanged).  One 4-D
// TMA box brings the CTA's halo patch (n rows x TX*m+2 columns x G channels;
// outside the image the box reads zeros, which is the pad-1 border) into
// shared memory.  V goes to shared memory in batches of taps (half of them for
// F(6,3), all of them for the smaller tiles), a [tap][64 channels] block per
// warp (rows of 72 words, the second chunk at word 36: conflict-free 16-byte reads); the lanes then
// take the batch's (tap, 32-channel chunk) items in turn: the chunk's absmax
// (the two chunks of a G=64 group combine across a lane pair, G >= 128 across
// warps in shared memory), the group scale, and 32 codes (quant4), written as
// two 16-byte stores of the tap-major Vq.
// Layers with few tiles per channel group run a split kernel instead (below):
// one thread per (tile, channel pair, batch of two rows of V), same chains.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace wino {
namespace {

template <typename T>
struct Pair;
template <>
struct Pair<uint16_t> {   // bf16 x 2 -> fp32 x 2 (exact)
    static __device__ __forceinline__ uint64_t load(const uint16_t* p) {
        const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
        return f2_pack(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
    }
};
template <>
struct Pair<float> {
    static __device__ __forceinline__ uint64_t load(const float* p) { return *reinterpret_cast<const uint64_t*>(p); }
};

// V staging rows in shared memory: chunk 0 at word 0, chunk 1 at word 36 (so the two chunk rows
// of one tap start on different banks), pitch 72 (8 taps x 2 chunks of float4 reads per quarter
// warp hit 32 distinct banks)
constexpr int kVPitch = 72, kVChunk1 = 36;

template <int M, typename Tin, int G>
struct InCfg {
    static constexpr int N = M + 2, N2 = N * N;
    static constexpr int NB = M == 6 ? 2 : 1;          // batches of taps staged in shared memory
    static constexpr int TB = N2 / NB, RB = N / NB;    // taps and transform rows per batch
    static constexpr int kMaxThreads = 160;   // measured: up to 10 tiles of G=32 per CTA
    static constexpr int kPitch = kVPitch, kChunk1 = kVChunk1;
    static constexpr int kMaxWarps = kMaxThreads / 32;
    __host__ __device__ static size_t patch_bytes(int tx) { return sizeof(Tin) * N * (size_t)(tx * M + 2) * G; }
    __host__ __device__ static int threads(int tx) { return (tx * (G / 2) + 31) / 32 * 32; }
    // the V blocks reuse the patch's shared memory once every thread holds its patch values
    __host__ __device__ static size_t smem(int tx) {
        const size_t v = sizeof(float) * (threads(tx) / 32) * TB * kPitch;
        return patch_bytes(tx) > v ? patch_bytes(tx) : v;
    }
};

// Items (tap, 32-channel chunk) of one batch of TB taps staged by one warp in vw ([TB][kPitch],
// chunk 1 at word kChunk1), one per lane and round: absmax of the chunk's 32 channels, the group
// maximum (G = 64: the two chunks of a tap sit on lanes 2k and 2k+1; G > 64: across CPW warps in
// shared memory), the scale and 32 codes, stored 16 B at a time.  lwarp is the warp's index among
// the warps that own the CTA's (tile, channel pair) threads for this batch.
template <int G, int TB, int MAXW>
__device__ __forceinline__ void quant_batch(const float* vw, int lane, int warp, int lwarp, int tap0, int TX,
                                            int tx0, int row_id, int g, const InputArgs& p, float (&red)[MAXW][TB]) {
    constexpr int P = kVPitch, C1 = kVChunk1;
    constexpr int CPW = G <= 64 ? 1 : G / 64;    // warps per group (G > 64)
    // a chunk's 32 codes start at a multiple of 32 bytes of a row of Cin (a multiple of 32) bytes, so
    // they fill one sector whenever the Vq base is 32-byte aligned (the workspace is promised 16)
    const bool vq_v8 = (reinterpret_cast<uintptr_t>(p.Vq) & 31u) == 0;
#pragma unroll
    for (int r0 = 0; r0 < 2 * TB; r0 += 32) {
        const int k = r0 + lane;
        const bool own = k < 2 * TB;
        const int tl_ = own ? k >> 1 : 0, c = k & 1;
        const int tap = tap0 + tl_;
        const float4* row = reinterpret_cast<const float4*>(vw + tl_ * P + C1 * c);
        float am = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x4 = row[j];
            am = max_abs3(am, x4.x, x4.y);
            am = max_abs3(am, x4.z, x4.w);
        }
        if (!own) am = 0.0f;
        if (G >= 64) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        if (G > 64) {
            if (c == 0 && own) red[warp][tl_] = am;
            __syncthreads();
            const int leader = warp - warp % CPW;
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < CPW; ++i) a = fmaxf(a, red[leader + i][tl_]);
            am = a;
            __syncthreads();   // red is reused by the next round
        }
        const int th = lwarp * 32 + 16 * c;    // first thread of the chunk (within its batch group)
        const int ctl = th / (G / 2);          // its tile
        const int ch = 2 * (th % (G / 2));     // its first channel within the group
        const int tx = tx0 + ctl;
        if (!own || ctl >= TX || tx >= p.TW) continue;
        const long t = (long)row_id * p.TW + tx;
        const QScale q = make_qscale(am);
        const size_t si = ((size_t)tap * (p.Cin / G) + g) * p.T_pad + t;
        if (ch == 0 && in_bounds(si, p.n_sv, p.err)) p.sV[si] = q.s;
        uint32_t w[8];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // two 16-value halves of the chunk, one exactness check each
            float xv[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 x4 = row[4 * hh + j];
                xv[4 * j] = x4.x;
                xv[4 * j + 1] = x4.y;
                xv[4 * j + 2] = x4.z;
                xv[4 * j + 3] = x4.w;
            }
            uint32_t wh[4];
            quant_chunk<16>(xv, q, wh);
#pragma unroll
            for (int j = 0; j < 4; ++j) w[4 * hh + j] = wh[j];
        }
        const size_t vi = ((size_t)tap * p.T_pad + t) * p.Cin + g * G + ch;
        if (!in_bounds(vi + 31, p.n_vq, p.err)) continue;
        if (vq_v8) {   // the chunk's 32 codes as one whole 32-byte sector
            sm100::st_global_v8(reinterpret_cast<uint32_t*>(p.Vq + vi), w);
        } else {
            uint4* dst = reinterpret_cast<uint4*>(p.Vq + vi);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

template <int M, uint64_t MASK, typename Tin, int G>
// at most 128 registers: three CTAs of a 10-tile row (160 threads) share an SM (measured best;
// the few spilled bytes cost less than the lost occupancy)
__global__ void __maxnreg__(MASK == kMaskAll ? 255 : 128)
    input_transform_kernel(const __grid_constant__ CUtensorMap tmX, InputArgs p, TransformArgs tf, int TX) {
    using Cfg = InCfg<M, Tin, G>;
    constexpr int N = M + 2, P = Cfg::kPitch, C1 = Cfg::kChunk1, NB = Cfg::NB, TB = Cfg::TB, RB = Cfg::RB;
    extern __shared__ __align__(128) unsigned char smem[];
    const Tin* patch = reinterpret_cast<const Tin*>(smem);   // [N][PW][G]
    float* vbuf = reinterpret_cast<float*>(smem);             // [warps][TB][P], after the patch is consumed
    __shared__ float red[Cfg::kMaxWarps][TB];
    __shared__ uint64_t bar;
    __shared__ int load_ok;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_dependents_launch();
    grid_dependency_wait();
    const int PW = TX * M + 2;
    const int row_id = blockIdx.y;  // img * TH + ty
    const int img = row_id / p.TH, ty = row_id - img * p.TH;
    const int tx0 = blockIdx.x * TX;
    const int g = blockIdx.z;

    if (tid == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        sm100::mbar_arrive_expect_tx(&bar, (uint32_t)Cfg::patch_bytes(TX));
        sm100::tma_load_4d(smem, &tmX, &bar, g * G, tx0 * M - 1, ty * M - 1, img);
    }
    if (g == 0)
        for (int i = tid; i < TX * p.ngo; i += blockDim.x) {
            const int tt = i / p.ngo, k = i - tt * p.ngo;
            const size_t ai = ((size_t)row_id * p.TW + tx0 + tt) * p.ngo + k;
            if (tx0 + tt < p.TW && in_bounds(ai, p.n_amax, p.err)) p.amax[ai] = 0u;
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

    // 1. this thread's tile and channel pair (threads past the CTA's tiles read tile 0 and store nothing)
    const int tl = tid / (G / 2) < TX ? tid / (G / 2) : 0;   // tile within the CTA
    const int cp = 2 * (tid % (G / 2));                       // first channel of the pair within the group
    uint64_t v[N][N];
#pragma unroll
    for (int r = 0; r < N; ++r)
#pragma unroll
        for (int l = 0; l < N; ++l) v[r][l] = Pair<Tin>::load(patch + (r * PW + tl * M + l) * G + cp);
    __syncthreads();   // the patch is consumed; its shared memory now holds the V blocks
    // 2. T1 = B^T d, in place, column by column
#pragma unroll
    for (int l = 0; l < N; ++l) {
        uint64_t tcol[N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            uint64_t acc = 0ull;
#pragma unroll
            for (int k = 0; k < N; ++k)
                if ((MASK >> (i * N + k)) & 1ull) acc = f2_fma(tf.BTd[i * N + k], v[k][l], acc);
            tcol[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) v[i][l] = tcol[i];
    }
    float* vw = vbuf + (size_t)warp * TB * P;
#pragma unroll
    for (int h = 0; h < NB; ++h) {
        // 3. V = T1 B for the rows of this batch: taps h*TB .. h*TB + TB - 1
        if (h) __syncwarp();   // the previous batch's codes are written
#pragma unroll
        for (int i = h * RB; i < (h + 1) * RB; ++i) {
#pragma unroll
            for (int j = 0; j < N; ++j) {
                uint64_t acc = 0ull;
#pragma unroll
                for (int l = 0; l < N; ++l)
                    if ((MASK >> (j * N + l)) & 1ull) acc = f2_fma(v[i][l], tf.BTd[j * N + l], acc);
                *reinterpret_cast<uint64_t*>(vw + (i * N + j - h * TB) * P + 2 * lane + (lane >= 16 ? C1 - 32 : 0)) = acc;
            }
        }
        __syncwarp();

        // 4.-5. items (tap, chunk) of the batch
        quant_batch<G, TB, Cfg::kMaxWarps>(vw, lane, warp, warp, h * TB, TX, tx0, row_id, g, p, red);
    }
}

// ----------------------------------------------------------------------------
// Layers with few tiles per channel group (small images, many channels): the grid above then
// holds too few threads to hide latency.  The split kernel gives every (tile, channel pair) NB
// threads, one per batch of RB rows of V: thread h forms rows h*RB .. h*RB + RB - 1 of
// T1 = B^T d and of V = T1 B, reading d from the shared-memory patch column by column -- T1[i][l]
// is its fma chain over k and V[i][j] takes its term l in ascending l, the chains of the two full
// passes -- and its warp quantises those rows' taps.
template <int M, typename Tin, int G>
struct InSplitCfg {
    static constexpr int N = M + 2;
    static constexpr int NB = M == 6 ? 4 : (M == 4 ? 3 : 2);   // row batches = threads per item
    static constexpr int RB = N / NB, TB = RB * N;              // rows and taps per batch
    static constexpr int kMaxThreads = 512, kMaxWarps = kMaxThreads / 32;
    __host__ __device__ static size_t patch_bytes(int tx) { return sizeof(Tin) * N * (size_t)(tx * M + 2) * G; }
    __host__ __device__ static int tpb(int tx) { return (tx * (G / 2) + 31) / 32 * 32; }   // threads per batch
    __host__ __device__ static int threads(int tx) { return NB * tpb(tx); }
    // the patch stays in place for every batch; the V blocks follow it
    __host__ __device__ static size_t vbuf_offset(int tx) { return (patch_bytes(tx) + 127) / 128 * 128; }
    __host__ __device__ static size_t smem(int tx) {
        return vbuf_offset(tx) + sizeof(float) * (threads(tx) / 32) * TB * kVPitch;
    }
};

template <int M, uint64_t MASK, typename Tin, int G, int H>
__device__ __forceinline__ void split_rows(const Tin* pt, int PW, const TransformArgs& tf, float* vw, int lane) {
    using Cfg = InSplitCfg<M, Tin, G>;
    constexpr int N = M + 2, RB = Cfg::RB;
    uint64_t vacc[RB][N];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int j = 0; j < N; ++j) vacc[r][j] = 0ull;
#pragma unroll
    for (int l = 0; l < N; ++l) {
        uint64_t dcol[N];
#pragma unroll
        for (int k = 0; k < N; ++k) {
            bool used = false;
#pragma unroll
            for (int r = 0; r < RB; ++r) used |= ((MASK >> ((H * RB + r) * N + k)) & 1ull) != 0;
            dcol[k] = used ? Pair<Tin>::load(pt + (size_t)(k * PW + l) * G) : 0ull;
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int i = H * RB + r;
            uint64_t t1 = 0ull;
#pragma unroll
            for (int k = 0; k < N; ++k)
                if ((MASK >> (i * N + k)) & 1ull) t1 = f2_fma(tf.BTd[i * N + k], dcol[k], t1);
#pragma unroll
            for (int j = 0; j < N; ++j)
                if ((MASK >> (j * N + l)) & 1ull) vacc[r][j] = f2_fma(t1, tf.BTd[j * N + l], vacc[r][j]);
        }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int j = 0; j < N; ++j)
            *reinterpret_cast<uint64_t*>(vw + (r * N + j) * kVPitch + 2 * lane + (lane >= 16 ? kVChunk1 - 32 : 0)) =
                vacc[r][j];
}

template <int M, uint64_t MASK, typename Tin, int G>
__global__ void __launch_bounds__(InSplitCfg<M, Tin, G>::kMaxThreads)
    input_transform_split_kernel(const __grid_constant__ CUtensorMap tmX, InputArgs p, TransformArgs tf, int TX) {
    using Cfg = InSplitCfg<M, Tin, G>;
    constexpr int NB = Cfg::NB, TB = Cfg::TB;
    extern __shared__ __align__(128) unsigned char smem[];
    const Tin* patch = reinterpret_cast<const Tin*>(smem);                    // [N][PW][G]
    float* vbuf = reinterpret_cast<float*>(smem + Cfg::vbuf_offset(TX));     // [warps][TB][kVPitch]
    __shared__ float red[Cfg::kMaxWarps][TB];
    __shared__ uint64_t bar;
    __shared__ int load_ok;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_dependents_launch();
    grid_dependency_wait();
    const int PW = TX * M + 2;
    const int row_id = blockIdx.y;  // img * TH + ty
    const int img = row_id / p.TH, ty = row_id - img * p.TH;
    const int tx0 = blockIdx.x * TX;
    const int g = blockIdx.z;

    if (tid == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        sm100::mbar_arrive_expect_tx(&bar, (uint32_t)Cfg::patch_bytes(TX));
        sm100::tma_load_4d(smem, &tmX, &bar, g * G, tx0 * M - 1, ty * M - 1, img);
    }
    if (g == 0)
        for (int i = tid; i < TX * p.ngo; i += blockDim.x) {
            const int tt = i / p.ngo, k = i - tt * p.ngo;
            const size_t ai = ((size_t)row_id * p.TW + tx0 + tt) * p.ngo + k;
            if (tx0 + tt < p.TW && in_bounds(ai, p.n_amax, p.err)) p.amax[ai] = 0u;
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

    // this thread's batch, tile and channel pair (threads past the CTA's tiles read tile 0 and store nothing)
    const int tpb = Cfg::tpb(TX);
    const int h = tid / tpb, ltid = tid - h * tpb, lwarp = ltid >> 5;
    const int tl = ltid / (G / 2) < TX ? ltid / (G / 2) : 0;
    const int cp = 2 * (ltid % (G / 2));
    const Tin* pt = patch + (size_t)(tl * M) * G + cp;   // d[k][l] at pt[(k * PW + l) * G]
    float* vw = vbuf + (size_t)warp * TB * kVPitch;
    if (h == 0) split_rows<M, MASK, Tin, G, 0>(pt, PW, tf, vw, lane);
    else if (h == 1) split_rows<M, MASK, Tin, G, 1>(pt, PW, tf, vw, lane);
    else if constexpr (NB > 2) {
        if (h == 2) split_rows<M, MASK, Tin, G, 2 % NB>(pt, PW, tf, vw, lane);
        else if constexpr (NB > 3) split_rows<M, MASK, Tin, G, 3 % NB>(pt, PW, tf, vw, lane);
    }
    __syncwarp();
    quant_batch<G, TB, Cfg::kMaxWarps>(vw, lane, warp, lwarp, h * TB, TX, tx0, row_id, g, p, red);
}

// Below a resident wave of the grid above (three 160-thread CTAs per SM) the split kernel runs.
inline long split_in_threads(int num_sms) { return (long)num_sms * 3 * 160; }

template <int M, uint64_t MASK, typename Tin, int G>
cudaError_t launch_split_g(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    using Cfg = InSplitCfg<M, Tin, G>;
    const int max_tx = std::max(1, std::min(Cfg::kMaxThreads / Cfg::NB / (G / 2), (256 - 2) / M));
    const int nblk = (a.TW + max_tx - 1) / max_tx;
    const int TX = (a.TW + nblk - 1) / nblk;
    CUtensorMap tm;
    const cuuint64_t es = sizeof(Tin);
    const cuuint64_t dims[4] = {(cuuint64_t)a.Cin, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.N};
    const cuuint64_t strides[3] = {es * a.Cin, es * a.Cin * a.W, es * a.Cin * a.W * a.H};
    const cuuint32_t box[4] = {(cuuint32_t)G, (cuuint32_t)(TX * M + 2), (cuuint32_t)Cfg::N, 1u};
    if (!make_tensor_map(&tm, sizeof(Tin) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                         a.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = input_transform_split_kernel<M, MASK, Tin, G>;
    const size_t smem = Cfg::smem(TX);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(nblk, a.N * a.TH, a.Cin / G);
    return launch_dependent(kern, grid, dim3(Cfg::threads(TX)), smem, st, tm, a, tf, TX);
}

}  // namespace

bool input_transform_split(int m, int G, int N, int TH, int TW, int Cin, int num_sms) {
    // the choice launch_g makes: tiles per CTA as there (at most 160 threads), then the grid size
    const int max_tx = std::min(160 / (G / 2), (256 - 2) / m);
    const int nblk = (TW + max_tx - 1) / max_tx;
    const int TX = (TW + nblk - 1) / nblk;
    const long threads = (TX * (G / 2) + 31) / 32 * 32;
    return (long)nblk * N * TH * (Cin / G) * threads < split_in_threads(num_sms);
}

namespace {

template <int M, uint64_t MASK, typename Tin, int G>
cudaError_t launch_g(const InputArgs& a, const TransformArgs& tf, cudaStream_t st) {
    using Cfg = InCfg<M, Tin, G>;
    // tiles per CTA: the whole tile row when it fits, else the row split into equal shares
    const int max_tx = std::min(Cfg::kMaxThreads / (G / 2), (256 - 2) / M);
    const int nblk = (a.TW + max_tx - 1) / max_tx;
    const int TX = (a.TW + nblk - 1) / nblk;
    static_assert(Cfg::kMaxThreads == 160, "input_transform_split mirrors this configuration");
    if (input_transform_split(M, G, a.N, a.TH, a.TW, a.Cin, a.num_sms)) return launch_split_g<M, MASK, Tin, G>(a, tf, st);
    // x [N][H][W][Cin] as a 4-D tensor (Cin, W, H, N); box G x (TX*m+2) x n x 1
    CUtensorMap tm;
    const cuuint64_t es = sizeof(Tin);
    const cuuint64_t dims[4] = {(cuuint64_t)a.Cin, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.N};
    const cuuint64_t strides[3] = {es * a.Cin, es * a.Cin * a.W, es * a.Cin * a.W * a.H};
    const cuuint32_t box[4] = {(cuuint32_t)G, (cuuint32_t)(TX * M + 2), (cuuint32_t)Cfg::N, 1u};
    if (!make_tensor_map(&tm, sizeof(Tin) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                         a.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = input_transform_kernel<M, MASK, Tin, G>;
    const size_t smem = Cfg::smem(TX);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(nblk, a.N * a.TH, a.Cin / G);
    return launch_dependent(kern, grid, dim3(Cfg::threads(TX)), smem, st, tm, a, tf, TX);
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
    if (m == 2) {
        if (bf16_in)
            return masked ? launch_cc<2, kMaskBT_F2, uint16_t>(a, tf, st) : launch_cc<2, kMaskAll, uint16_t>(a, tf, st);
        return masked ? launch_cc<2, kMaskBT_F2, float>(a, tf, st) : launch_cc<2, kMaskAll, float>(a, tf, st);
    }
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
