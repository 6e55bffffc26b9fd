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
// pairs: every tap load and output store of a warp is contiguous.  Column nu
// of Z is formed from column nu of Y and at once added into every output
// o[i][j] (whose chain over nu stays in ascending order), so only the output
// tile and one column are live.
// Variants: per-tap Y groups (the Y_TAP reading), and, for layers with few
// (tile, channel pair) items on the fp32-Y path, a split kernel with N threads
// per item (one per column of Y, then one per output row).
#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

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

// Bounded wait for a phase of one column slot's TMA barrier (records a timeout in the error word).
__device__ __forceinline__ bool column_wait(uint64_t* bar, uint32_t parity, int* err) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = sm100::globaltimer();
    while (!sm100::mbar_try_wait(bar, parity))
        if (sm100::globaltimer() - t0 > sm100::kWaitLimitNs) {
            atomicCAS(err, 0, sm100::kDevErrTimeout);
            return false;
        }
    return true;
}

constexpr int kYRing = 4;   // column slots of the fp32 source: 4 x 8 KiB for F(6,3), four CTAs per SM

template <int M, uint64_t MASK, bool SRC_Y32, bool BF16_OUT, bool DEBUG>
__global__ void __launch_bounds__(128, 4)
    output_transform_kernel(const __grid_constant__ CUtensorMap tmY, OutputArgs p, TransformArgs tf) {
    constexpr int N = M + 2, N2 = N * N;
    // The CTA's 128 cout pairs are 256 consecutive elements of every tap's [T][Cout] plane.  One 3-D
    // TMA box per column nu of Y (taps xi * N + nu, every xi) brings them to shared memory as
    // [xi][256], each column slot on its own barrier.  The int8 source keeps every column (256 bytes
    // per tap, static); the fp32 source cycles R = kYRing slots (1 KiB per tap, dynamic): once every
    // thread has read column nu, its slot is refilled with column nu + R, so the transform of the
    // first columns overlaps the later columns' loads and a CTA holds 4 columns instead of N.
    constexpr int R = (SRC_Y32 && kYRing < N) ? kYRing : N;
    constexpr uint32_t kColBytes = (SRC_Y32 ? 1024u : 256u) * N;
    __shared__ __align__(128) uint8_t ysm[SRC_Y32 ? 16 : 256 * N2];
    extern __shared__ __align__(128) unsigned char ydyn[];
    unsigned char* ybuf = SRC_Y32 ? ydyn : ysm;
    __shared__ uint64_t bar[R];
    grid_dependents_launch();
    grid_dependency_wait();
    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) sm100::mbar_init(&bar[s], 1);
        sm100::fence_mbar_init();
        for (int nu = 0; nu < R; ++nu) {
            sm100::mbar_arrive_expect_tx(&bar[nu], kColBytes);
            sm100::tma_load_3d(ybuf + (size_t)nu * kColBytes, &tmY, &bar[nu], (int)(blockIdx.x * 256u), nu, 0);
        }
    }
    __syncthreads();
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const int cpairs = p.Cout >> 1;
    const long t = i / cpairs;
    const int co = 2 * (int)(i - t * cpairs);
    const int cg = co / p.G;
    const size_t base = (size_t)t * p.Cout + co;   // Yq / Y32 are tap-major [n2][T][Cout]
    const size_t tstride = (size_t)p.T * p.Cout;
    // every Y element this thread touches lies in [base, base + (N2 - 1) * tstride + 1]; a thread
    // past the last tile (or failing a debug-build index check) still takes part in the ring
    const bool active = t < p.T && in_bounds((size_t)t * p.ngo + cg, p.n_amax, p.err) &&
                        (!(SRC_Y32 || DEBUG) || in_bounds(base + (size_t)(N2 - 1) * tstride + 1, p.n_y, p.err)) &&
                        (!DEBUG || in_bounds((size_t)t * p.ngo + cg, p.n_sy, p.err));
    const QScale qs = make_qscale(active ? __uint_as_float(p.amax[(size_t)t * p.ngo + cg]) : 0.0f);
    if (DEBUG && active && co % p.G == 0) p.sY_dbg[(size_t)t * p.ngo + cg] = qs.s;
    const uint64_t s2 = f2_pack(qs.s, qs.s);

    // o[r][c] = fma chain over ascending nu of Z[r][nu] * AT[c][nu], with Z[r][nu] = fma chain over
    // ascending xi of AT[r][xi] * Yd[xi][nu]: column nu of Z is formed and used at once, so only the
    // output tile (M x M pairs) and one column stay live
    uint64_t o[M][M];
#pragma unroll
    for (int r = 0; r < M; ++r)
#pragma unroll
        for (int c = 0; c < M; ++c) o[r][c] = 0ull;
    bool ok = true;
#pragma unroll
    for (int nu = 0; nu < N; ++nu) {
        const int slot = nu % R;
        if (ok && !column_wait(&bar[slot], (uint32_t)((nu / R) & 1), p.err)) ok = false;
        uint64_t Yc[N];                            // column nu of Yd: taps xi * N + nu
        if (SRC_Y32) {
            const float* ys = reinterpret_cast<const float*>(ybuf + (size_t)slot * kColBytes) + 2 * threadIdx.x;
#pragma unroll
            for (int xi = 0; xi < N; xi += 2) {
                const float2 a = *reinterpret_cast<const float2*>(ys + xi * 256);
                const float2 b = *reinterpret_cast<const float2*>(ys + (xi + 1) * 256);
                const Quad qd = quant4(a.x, a.y, b.x, b.y, qs);
                Yc[xi] = f2_mul(s2, qd.k01);
                Yc[xi + 1] = f2_mul(s2, qd.k23);
                if (DEBUG && active) {
                    *reinterpret_cast<uint16_t*>(p.Yq_dbg + base + (size_t)(xi * N + nu) * tstride) =
                        (uint16_t)(qd.packed & 0xffffu);
                    *reinterpret_cast<uint16_t*>(p.Yq_dbg + base + (size_t)((xi + 1) * N + nu) * tstride) =
                        (uint16_t)(qd.packed >> 16);
                }
            }
            if (nu + R < N) {   // every thread has read the slot: refill it with column nu + R
                __syncthreads();
                if (threadIdx.x == 0 && ok) {
                    sm100::fence_proxy_async_smem();
                    sm100::mbar_arrive_expect_tx(&bar[slot], kColBytes);
                    sm100::tma_load_3d(ybuf + (size_t)slot * kColBytes, &tmY, &bar[slot], (int)(blockIdx.x * 256u),
                                       nu + R, 0);
                }
            }
        } else {
#pragma unroll
            for (int xi = 0; xi < N; ++xi) {
                const uint32_t x = *reinterpret_cast<const uint16_t*>(ybuf + (size_t)slot * kColBytes + xi * 256 +
                                                                       2 * threadIdx.x);
                Yc[xi] = f2_mul(s2, codes2_to_f2(x));
            }
        }
#pragma unroll
        for (int r = 0; r < M; ++r) {
            uint64_t z = 0ull;
#pragma unroll
            for (int xi = 0; xi < N; ++xi)
                if ((MASK >> (r * N + xi)) & 1ull) z = f2_fma(tf.ATd[r * N + xi], Yc[xi], z);
#pragma unroll
            for (int c = 0; c < M; ++c)
                if ((MASK >> (c * N + nu)) & 1ull) o[r][c] = f2_fma(z, tf.ATd[c * N + nu], o[r][c]);
        }
    }
    if (!active || !ok) return;
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
            float o0, o1;
            f2_unpack(o[r][c], o0, o1);
            const size_t oi = (((size_t)img * p.H + yy) * p.W + xx) * p.Cout + co;
            if (!in_bounds(oi + 1, p.n_out, p.err)) continue;
            if (BF16_OUT)
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p.out) + oi) =
                    __floats2bfloat162_rn(o0, o1);
            else
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + oi) = make_float2(o0, o1);
        }
    }
}

// Per-tap Y groups (the Y_TAP reading): Y is requantised with one scale per
// (tile, tap, G couts).  Same thread layout as output_transform_kernel, fp32 Y
// source only.  Pass 1 reduces each tap's |Y| over the group -- the G/2 lanes of
// a warp segment by shuffles, or (G >= 128) the G/64 warps of the CTA through
// shared memory -- and one thread per (group, tap) stores the scale; pass 2 is
// the fp32-Y path of output_transform_kernel with the tap's own scale.
template <int M, uint64_t MASK, bool BF16_OUT>
__global__ void __launch_bounds__(128, 6) output_transform_ytap_kernel(OutputArgs p, TransformArgs tf) {
    constexpr int N = M + 2, N2 = N * N;
    __shared__ QScale qsm[4][2][N2];     // [warp][segment][tap] (G <= 64) or [group in CTA][0][tap]
    __shared__ float red[4][2][N2];      // per-warp (and segment) maxima
    grid_dependents_launch();
    grid_dependency_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const int cpairs = p.Cout >> 1;
    const long t = i / cpairs;
    const int co = 2 * (int)(i - t * cpairs);
    // a CTA covers whole groups; dead threads (and, in the debug build, threads whose Y range fails
    // its index check) still join the reductions with zeros
    const bool live = t < p.T && in_bounds(((size_t)t * p.Cout + co) + (size_t)(N2 - 1) * p.T * p.Cout + 1,
                                           p.n_y, p.err);
    const int G = p.G;
    const int cg = co / G;
    const size_t base = (size_t)(live ? t : 0) * p.Cout + co;
    const size_t tstride = (size_t)p.T * p.Cout;

    // ---- pass 1: per-tap group scales.  Eight taps at a time: their loads in flight together
    // and their lane reductions interleaved; the segment's first lane keeps the maxima.
    const int seg_w = G <= 64 ? G / 2 : 32;        // lanes of the warp reduced together
    const int seg = lane / seg_w, sl = lane % seg_w;
    for (int t0 = 0; t0 < N2; t0 += 8) {
        float a[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            a[k] = 0.0f;
            if (live && t0 + k < N2) {
                const float2 y = *reinterpret_cast<const float2*>(p.Y32 + base + (size_t)(t0 + k) * tstride);
                a[k] = fmaxf(fabsf(y.x), fabsf(y.y));
            }
        }
        for (int o = seg_w / 2; o > 0; o >>= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], __shfl_xor_sync(0xffffffffu, a[k], o));
        if (sl == 0)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (t0 + k < N2) red[warp][seg][t0 + k] = a[k];
    }
    if (G <= 64) {
        __syncwarp();
        // each lane of the segment derives the scales of every seg_w-th tap
        for (int tap = sl; tap < N2; tap += seg_w) {
            qsm[warp][seg][tap] = make_qscale(red[warp][seg][tap]);
            const size_t di = ((size_t)t * N2 + tap) * p.ngo + cg;
            if (p.sY_dbg && live && in_bounds(di, p.n_sy, p.err)) p.sY_dbg[di] = qsm[warp][seg][tap].s;
        }
        __syncwarp();
    } else {
        __syncthreads();
        const int wpg = G / 64;                    // warps per group
        const int ngc = 4 / wpg;                   // groups in the CTA
        for (int k = threadIdx.x; k < ngc * N2; k += blockDim.x) {
            const int gi = k / N2, tap = k % N2;
            float a = 0.0f;
            for (int w = 0; w < wpg; ++w) a = fmaxf(a, red[gi * wpg + w][0][tap]);
            qsm[gi][0][tap] = make_qscale(a);
            const long i0 = (long)blockIdx.x * blockDim.x + gi * (G / 2);   // first thread of the group
            const long tg = i0 / cpairs;
            const size_t di = ((size_t)tg * N2 + tap) * p.ngo + (int)(i0 - tg * cpairs) * 2 / G;
            if (p.sY_dbg && tg < p.T && in_bounds(di, p.n_sy, p.err)) p.sY_dbg[di] = qsm[gi][0][tap].s;
        }
        __syncthreads();
    }
    if (!live) return;
    const QScale* myq = G <= 64 ? qsm[warp][lane / (G / 2)] : qsm[warp / (G / 64)][0];

    // ---- pass 2: requantise with the tap's scale, then A^T . A
    uint64_t Z[M][N];
#pragma unroll
    for (int nu = 0; nu < N; ++nu) {
        uint64_t Yc[N];
#pragma unroll
        for (int xi = 0; xi < N; ++xi) {
            const int tap = xi * N + nu;
            const QScale q = myq[tap];
            const float2 y = *reinterpret_cast<const float2*>(p.Y32 + base + (size_t)tap * tstride);
            const Quad qd = quant4(y.x, y.y, y.x, y.y, q);
            Yc[xi] = f2_mul(f2_pack(q.s, q.s), qd.k01);
            if (p.Yq_dbg)
                *reinterpret_cast<uint16_t*>(p.Yq_dbg + base + (size_t)tap * tstride) = (uint16_t)(qd.packed & 0xffffu);
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
            if (!in_bounds(o + 1, p.n_out, p.err)) continue;
            if (BF16_OUT)
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p.out) + o) =
                    __floats2bfloat162_rn(o0, o1);
            else
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + o) = make_float2(o0, o1);
        }
    }
}

// Layers with few (tile, channel pair) items -- too few for one thread each to fill the GPU --
// on the fp32-Y path: N threads per item, one per column nu of Y.  Thread nu requantises its
// column's N taps and forms column nu of Z = A^T Yd; after a warp barrier thread r < M forms
// output row r from row r of Z.  The arithmetic and every chain order are those of
// output_transform_kernel; each thread's chain is an N-th as long.
template <int M, uint64_t MASK, bool BF16_OUT, bool DEBUG>
__global__ void __launch_bounds__(128) output_transform_split_kernel(OutputArgs p, TransformArgs tf) {
    constexpr int N = M + 2;
    constexpr int IPW = 32 / N;                   // items per warp (F(4,3): lanes 30, 31 idle)
    __shared__ uint64_t zs[4][IPW][M][N];         // Z of each item, (co, co + 1) pairs
    grid_dependents_launch();
    grid_dependency_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slot = lane / N, nu = lane - slot * N;
    const long item = ((long)blockIdx.x * 4 + warp) * IPW + slot;   // (tile, channel pair)
    const int cpairs = p.Cout >> 1;
    const long t = item / cpairs;
    const int co = 2 * (int)(item - t * cpairs);
    const bool live = slot < IPW && t < p.T &&
                      in_bounds((size_t)t * p.ngo + co / p.G, p.n_amax, p.err) &&
                      in_bounds((size_t)t * p.Cout + co + (size_t)(N * N - 1) * p.T * p.Cout + 1, p.n_y, p.err) &&
                      (!DEBUG || in_bounds((size_t)t * p.ngo + co / p.G, p.n_sy, p.err));
    if (live) {
        const int cg = co / p.G;
        const QScale qs = make_qscale(__uint_as_float(p.amax[(size_t)t * p.ngo + cg]));
        if (DEBUG && nu == 0 && co % p.G == 0) p.sY_dbg[(size_t)t * p.ngo + cg] = qs.s;
        const uint64_t s2 = f2_pack(qs.s, qs.s);
        const size_t base = (size_t)t * p.Cout + co;
        const size_t tstride = (size_t)p.T * p.Cout;
        uint64_t Yc[N];                           // column nu of Yd: taps xi * N + nu
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
#pragma unroll
        for (int r = 0; r < M; ++r) {
            uint64_t acc = 0ull;
#pragma unroll
            for (int xi = 0; xi < N; ++xi)
                if ((MASK >> (r * N + xi)) & 1ull) acc = f2_fma(tf.ATd[r * N + xi], Yc[xi], acc);
            zs[warp][slot][r][nu] = acc;
        }
    }
    __syncwarp();
    if (!live || nu >= M) return;
    const int r = nu;                             // this thread's output row
    const int TT = p.TH * p.TW;
    const int img = (int)(t / TT);
    const int rem = (int)(t - (long)img * TT);
    const int ty = rem / p.TW, tx = rem - ty * p.TW;
    const int yy = ty * M + r;
    if (yy >= p.H) return;
#pragma unroll
    for (int c = 0; c < M; ++c) {
        const int xx = tx * M + c;
        if (xx >= p.W) break;
        uint64_t acc = 0ull;
#pragma unroll
        for (int k = 0; k < N; ++k)
            if ((MASK >> (c * N + k)) & 1ull) acc = f2_fma(zs[warp][slot][r][k], tf.ATd[c * N + k], acc);
        float o0, o1;
        f2_unpack(acc, o0, o1);
        const size_t o = (((size_t)img * p.H + yy) * p.W + xx) * p.Cout + co;
        if (!in_bounds(o + 1, p.n_out, p.err)) continue;
        if (BF16_OUT)
            *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p.out) + o) =
                __floats2bfloat162_rn(o0, o1);
        else
            *reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + o) = make_float2(o0, o1);
    }
}

// Below two 128-thread CTAs' worth of (tile, channel pair) items per SM, the fp32-Y path splits
// each item over N threads.
inline long split_out_items(int num_sms) { return (long)num_sms * 2 * 128; }

}  // namespace

bool output_transform_split(long T, int Cout, bool src_y32, bool ytap, int num_sms) {
    return src_y32 && !ytap && T * (long)(Cout / 2) < split_out_items(num_sms);
}

namespace {

template <int M, uint64_t MASK>
cudaError_t launch_m(const OutputArgs& a, const TransformArgs& tf, bool src_y32, bool bf16_out, bool debug,
                     cudaStream_t st) {
    const long threads = a.T * (long)(a.Cout / 2);
    const dim3 grid((unsigned)((threads + 127) / 128));
    CUtensorMap tm;
    std::memset(&tm, 0, sizeof(tm));
    const bool split = output_transform_split(a.T, a.Cout, src_y32, a.ytap != 0, a.num_sms);
    if (!a.ytap && !split) {   // Yq / Y32 as [xi][nu][T*Cout]; box 256 x 1 x N (a CTA's 128 cout pairs, one column)
        const cuuint64_t es = src_y32 ? 4 : 1;
        const cuuint64_t n = (cuuint64_t)(M + 2);
        const cuuint64_t dims[3] = {(cuuint64_t)a.T * a.Cout, n, n};
        const cuuint64_t strides[2] = {(cuuint64_t)a.T * a.Cout * es, (cuuint64_t)a.T * a.Cout * es * n};
        const cuuint32_t box[3] = {256u, 1u, (cuuint32_t)n};
        if (!make_tensor_map(&tm, src_y32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                             src_y32 ? static_cast<const void*>(a.Y32) : static_cast<const void*>(a.Yq), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (a.ytap)
        return bf16_out ? launch_dependent(output_transform_ytap_kernel<M, MASK, true>, grid, dim3(128), 0, st, a, tf)
                        : launch_dependent(output_transform_ytap_kernel<M, MASK, false>, grid, dim3(128), 0, st, a, tf);
    if (split) {   // too few items for one thread each
        constexpr int IPW = 32 / (M + 2);
        const dim3 sgrid((unsigned)((threads + 4 * IPW - 1) / (4 * IPW)));
#define WINO_SPLIT_LAUNCH(BF, DBG) \
    return launch_dependent(output_transform_split_kernel<M, MASK, BF, DBG>, sgrid, dim3(128), 0, st, a, tf)
        if (bf16_out) {
            if (debug) WINO_SPLIT_LAUNCH(true, true); else WINO_SPLIT_LAUNCH(true, false);
        } else {
            if (debug) WINO_SPLIT_LAUNCH(false, true); else WINO_SPLIT_LAUNCH(false, false);
        }
#undef WINO_SPLIT_LAUNCH
    }
    // fp32 source: a ring of kYRing column slots of 1 KiB per tap (every column when there are fewer)
    const size_t dsmem = src_y32 ? (size_t)1024 * std::min(kYRing, M + 2) * (M + 2) : 0;
#define WINO_OUT_LAUNCH(Y32, BF, DBG)                                                                          \
    do {                                                                                                     \
        auto kern = output_transform_kernel<M, MASK, Y32, BF, DBG>;                                          \
        if (Y32) {                                                                                           \
            const cudaError_t fe = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                                        (int)dsmem);                                         \
            if (fe != cudaSuccess) return fe;                                                                \
        }                                                                                                    \
        return launch_dependent(kern, grid, dim3(128), dsmem, st, tm, a, tf);                                \
    } while (0)
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
