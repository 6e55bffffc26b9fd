// Fully fused group-wise int8 Winograd layer for small channel counts ("Data-Free
// Group-Wise Fully Quantized Winograd Convolution via Learnable Scales", Fig. 2:
// the input transform, the Hadamard product and the output transform are each
// group-wise quantised): one kernel takes x to the output, and neither the
// quantised input transform Vq nor the requantised Y ever leave the SM.
//
// Used for Cin, Cout in {32, 64} (their Vq and Yq of a 16-tile unit fit shared
// memory).  The arithmetic is that of the staged kernels, in the same order:
//   Vq, sV   V = B^T d B per (tile, channel) by the fp32 chains of the input
//            transform; Q over G consecutive channels at fixed (tile, tap);
//   Y        per tap, per K-group j the exact int32 dot product (tensor core),
//            y = fma((float)acc_j, RN(sV_j * sU_j), y) over ascending j;
//   sY, Yq   one scale per (tile, G output channels) over all n*n taps; Q;
//   out      A^T (sY * Yq) A by the output transform's chains, cropped.
//
// Persistent CTAs walk units of 16 consecutive tiles.  Per unit:
//   1. the compute warps load each tile's n x n patch (zeros outside the
//      image), transform it, reduce each (tap, group) maximum across the lanes
//      that hold the group, and write the int8 codes straight into the
//      tensor-core operand layout in shared memory (K-major, swizzle = Cin
//      bytes) together with the scales;
//   2. pass A: per tap an int8 MMA with swapped operands -- A = Uq[tap]
//      (128 rows = output channels, rows past Cout read as zeros by the TMA
//      box), B = the unit's Vq[tap] (16 tiles) -- into TMEM, one K-group per
//      accumulator; the epilogue dequantises and keeps |Y| maxima per (tile,
//      output channel group);
//   3. pass B: the same MMAs again; the epilogue requantises Y with sY and
//      writes int8 Yq to shared memory;
//   4. the output transform from shared memory to the NHWC output.
// Warp 0 streams Uq (4 taps per TMA stage), warp 1 allocates TMEM and issues
// the MMAs (one thread), warps 2..9 compute.  Every wait is bounded.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace wino {
namespace {

using namespace sm100;

constexpr int kFNT = 16;              // tiles per unit: the MMA's N (its M = 128 output-channel rows)
constexpr int kFTPS = 4;              // taps per Uq stage and per accumulator slot
constexpr int kFStages = 3;           // Uq stage ring
constexpr int kFComputeWarps = 8;
constexpr int kFThreads = 64 + 32 * kFComputeWarps;

template <typename T>
struct FPair;
template <>
struct FPair<uint16_t> {   // bf16 x 2 -> fp32 x 2 (exact)
    static __device__ __forceinline__ uint64_t load(const uint16_t* p) {
        const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
        return f2_pack(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
    }
};
template <>
struct FPair<float> {
    static __device__ __forceinline__ uint64_t load(const float* p) { return *reinterpret_cast<const uint64_t*>(p); }
};

template <int M, int CIN, int COUT, int G>
struct FCfg {
    static constexpr int N = M + 2, N2 = N * N;
    static constexpr int NGI = CIN / G, NGO = COUT / G;
    static constexpr int SEG = G / 2;                         // lanes holding one (tile, group): channel pairs
    static constexpr int VQ_TAP = kFNT * CIN;                 // bytes of one tap of the unit's Vq
    static constexpr int A_TAP = 128 * CIN;                   // one tap of Uq (rows past Cout are zeros)
    static constexpr int STAGE = kFTPS * A_TAP;
    static constexpr int SLOT_COLS = kFTPS * NGI * kFNT;      // TMEM columns per accumulator slot
    static constexpr int NSLOT = 512 / SLOT_COLS >= 4 ? 4 : 512 / SLOT_COLS;
    static constexpr int TMEM_COLS = SLOT_COLS * NSLOT <= 64 ? 64 : (SLOT_COLS * NSLOT <= 128 ? 128
                                     : (SLOT_COLS * NSLOT <= 256 ? 256 : 512));
    static constexpr int EPI_WARPS = 2 * (COUT / 32);          // compute warps whose TMEM lanes hold rows < Cout
    static constexpr int ROUNDS = CIN == 64 ? 2 : 1;          // transform rounds (8 or 16 tiles each)
    static constexpr int NSTEP = N2 / kFTPS;                  // Uq stages per pass (n*n is a multiple of 4)
    // shared memory carve-up (from a 1024-byte aligned base).  Yq of a tap takes the place of the
    // tap's Vq (same size, Cin = Cout): the second pass writes it only after that tap's MMAs, the
    // last readers of its Vq, have completed.
    static constexpr size_t OFF_VQ = 0;
    static constexpr size_t OFF_YQ = OFF_VQ;
    static constexpr size_t OFF_A = OFF_VQ + (size_t)N2 * VQ_TAP;
    static constexpr size_t OFF_SU = OFF_A + (size_t)kFStages * STAGE;   // [N2][NGI][COUT], once per CTA
    static constexpr size_t OFF_SV = OFF_SU + 4 * (size_t)N2 * NGI * COUT;
    static constexpr size_t OFF_QS = OFF_SV + 4 * (size_t)N2 * NGI * kFNT;
    static constexpr size_t OFF_AMAX = OFF_QS + 8 * (size_t)kFComputeWarps * 2 * 32;
    static constexpr size_t BYTES = OFF_AMAX + 4 * (size_t)kFNT * NGO;
    static_assert(N2 % kFTPS == 0, "whole stages of taps");
    static_assert(CIN % 32 == 0 && COUT % 32 == 0 && G % 32 == 0 && G <= CIN && G <= COUT, "shape");
    static_assert(CIN == COUT, "Yq reuses Vq's shared memory");
};

struct FRing {
    int idx;
    uint32_t phase;
    __device__ __forceinline__ void next(int n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

// Warp-uniform bounded wait: every lane polls, the loop exits for all lanes together.
__device__ __forceinline__ bool warp_wait_f(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        if ((it & 63u) == 63u) {
            bool stop = *abort_flag != 0;
            if (!stop && globaltimer() - t0 > kWaitLimitNs) {
                stop = true;
                *abort_flag = 1;
                atomicCAS(err, 0, kDevErrTimeout);
            }
            if (__any_sync(0xffffffffu, stop)) return false;
        }
    }
}

struct FTail {
    uint64_t a_full[kFStages];
    uint64_t a_empty[kFStages];
    uint64_t acc_full[4];
    uint64_t acc_empty[4];
    uint64_t vq_ready;
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
    int stop;   // uniform decision of the compute warps, written before and read after a barrier
};

// Byte offset of channel byte c of row r (a tile) within one tap of the K-major operand whose rows
// are CIN bytes and whose swizzle width is CIN bytes (the layout a TMA box of that swizzle writes):
// 8-row atoms of 8 * CIN bytes, the 16-byte chunk index XORed with row bits.
template <int CIN>
__device__ __forceinline__ int vq_offset(int r, int c) {
    const int r8 = r & 7;
    const int swz = CIN == 128 ? r8 : (CIN == 64 ? (r8 >> 1) & 3 : (r8 >> 2) & 1);
    return (r >> 3) * (8 * CIN) + r8 * CIN + ((((c >> 4) ^ swz) << 4) | (c & 15));
}

// Recursive-halving maximum over SEG lanes (16 or 32) of 32 values per lane: on return lane L holds
// in a[e], e < 32 / SEG, the maximum over its segment of entry (L % SEG) * (32 / SEG) + e.
template <int SEG>
__device__ __forceinline__ void seg_scatter_max32(float (&a)[32], int lane) {
    constexpr int STEPS = SEG == 32 ? 5 : 4;
#pragma unroll
    for (int step = 0; step < STEPS; ++step) {
        const int o = (SEG / 2) >> step;
        const int h = 16 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? a[i] : a[i + h];
            const float keep = upper ? a[i + h] : a[i];
            a[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
        }
    }
}

// Q for a pair of values sharing one scale (s, r = RN(1/s) or 0): the division-free fast path of
// quant4 with its fp64 fallback (RN53(1/s) derived there), codes as two bytes.
__device__ __forceinline__ uint32_t quant_pair(uint64_t v2, float s, float r) {
    if (r != 0.0f || s == 0.0f) {
        const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
        const uint64_t t = f2_mul(v2, f2_pack(r, r));
        const uint64_t a = f2_add(t, magic2);
        float d0, d1;
        f2_unpack(f2_sub(t, f2_sub(a, magic2)), d0, d1);
        if (fmaxf(fabsf(d0), fabsf(d1)) < 0.5f - 0x1p-12f) {
            float a0, a1;
            f2_unpack(a, a0, a1);
            return __byte_perm(__float_as_uint(a0), __float_as_uint(a1), 0x0040);
        }
    }
    QScale q;
    q.s = s;
    q.r = r;
    q.rd = s != 0.0f ? __drcp_rn((double)s) : 0.0;
    float v0, v1;
    f2_unpack(v2, v0, v1);
    return (uint32_t)(quant_code_fast(v0, q) & 0xff) | ((uint32_t)(quant_code_fast(v1, q) & 0xff) << 8);
}

// Q of one value with its own scale (fast path, fp64 fallback).
__device__ __forceinline__ int quant_one(float v, const QScale& q) {
    if (q.r != 0.0f || q.s == 0.0f) {
        const float t = __fmul_rn(v, q.r);
        const float a = __fadd_rn(t, kRoundMagic);
        if (fabsf(__fsub_rn(t, __fsub_rn(a, kRoundMagic))) < 0.5f - 0x1p-12f)
            return __float_as_int(a) - kRoundMagicBits;
    }
    return quant_code_fast(v, q);
}

__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kFComputeWarps) : "memory"); }

template <int M, uint64_t MBT, uint64_t MAT, typename Tin, int CIN, int COUT, int G>
__global__ void __launch_bounds__(kFThreads, 1)
    fused_small_kernel(const __grid_constant__ CUtensorMap tmU, FusedArgs p, TransformArgs tf) {
    using Cfg = FCfg<M, CIN, COUT, G>;
    const bool DEBUG = p.Vq_dbg != nullptr;   // debug copies of Vq, sV, Yq and sY
    const bool BF16_OUT = p.bf16_out != 0;
    constexpr int N = Cfg::N, N2 = Cfg::N2, NGI = Cfg::NGI, SEG = Cfg::SEG;
    extern __shared__ __align__(1024) unsigned char fsm_raw[];
    unsigned char* fsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(fsm_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* vq = fsm + Cfg::OFF_VQ;
    unsigned char* aring = fsm + Cfg::OFF_A;
    int8_t* yq = reinterpret_cast<int8_t*>(fsm + Cfg::OFF_YQ);
    float* sv = reinterpret_cast<float*>(fsm + Cfg::OFF_SV);            // [N2][NGI][kFNT]
    float* su_tab = reinterpret_cast<float*>(fsm + Cfg::OFF_SU);        // [N2][NGI][COUT]
    float2* qs_tab = reinterpret_cast<float2*>(fsm + Cfg::OFF_QS);      // [warp][2][32]: (s, r) per tap
    unsigned* amax = reinterpret_cast<unsigned*>(fsm + Cfg::OFF_AMAX);  // [kFNT][NGO] fp32 bits
    __shared__ FTail tail;
    volatile int* abort_flag = &tail.abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int units = (int)((p.T + kFNT - 1) / kFNT);
    grid_dependents_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(&tail.a_full[s], 1);
            mbar_init(&tail.a_empty[s], 1);
        }
        for (int b = 0; b < Cfg::NSLOT; ++b) {
            mbar_init(&tail.acc_full[b], 1);
            mbar_init(&tail.acc_empty[b], Cfg::EPI_WARPS);
        }
        mbar_init(&tail.vq_ready, 1);
        mbar_init(&tail.done, 1);
        tail.abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&tmU);
    }
    if (warp == 1) {
        tmem_alloc(&tail.tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    grid_dependency_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ Uq producer
        if (lane == 0) {
            FRing st{0, 0};
            uint32_t issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x)
                for (int pass = 0; ok && pass < 2; ++pass)
                    for (int s = 0; s < Cfg::NSTEP; ++s) {
                        if (!mbar_wait(&tail.a_empty[st.idx], st.phase ^ 1u, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&tail.a_full[st.idx], (uint32_t)Cfg::STAGE);
                        tma_load_3d(aring + (size_t)st.idx * Cfg::STAGE, &tmU, &tail.a_full[st.idx], 0, 0, s * kFTPS);
                        ++issued;
                        st.next(kFStages);
                    }
            FRing dr{st.idx, st.phase};   // drain: every issued load lands before the CTA exits
            for (uint32_t i = 0; i < issued && i < (uint32_t)kFStages; ++i) {
                if (dr.idx == 0) {
                    dr.idx = kFStages - 1;
                    dr.phase ^= 1u;
                } else {
                    --dr.idx;
                }
                mbar_wait_teardown(&tail.a_full[dr.idx], dr.phase);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(128, kFNT);
            FRing st{0, 0}, sl{0, 0};
            bool ok = true;
            uint32_t vq_phase = 0;
            for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
                ok = mbar_wait(&tail.vq_ready, vq_phase, abort_flag, p.err);
                vq_phase ^= 1u;
                tc_fence_after();
                for (int pass = 0; ok && pass < 2; ++pass)
                    for (int s = 0; s < Cfg::NSTEP; ++s) {
                        if (!mbar_wait(&tail.a_full[st.idx], st.phase, abort_flag, p.err) ||
                            !mbar_wait(&tail.acc_empty[sl.idx], sl.phase, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_base = smem_u32(aring + (size_t)st.idx * Cfg::STAGE);
                        const uint32_t d_slot = tmem_base + (uint32_t)(sl.idx * Cfg::SLOT_COLS);
#pragma unroll
                        for (int tt = 0; tt < kFTPS; ++tt) {
                            const int tap = s * kFTPS + tt;
                            const uint32_t a_tap = a_base + (uint32_t)(tt * Cfg::A_TAP);
                            const uint32_t b_tap = smem_u32(vq + (size_t)tap * Cfg::VQ_TAP);
#pragma unroll
                            for (int g = 0; g < NGI; ++g)
#pragma unroll
                                for (int k = 0; k < G / 32; ++k) {
                                    const uint32_t koff = (uint32_t)(g * G + 32 * k);
                                    mma_i8(d_slot + (uint32_t)((tt * NGI + g) * kFNT), smem_desc_kmajor(a_tap + koff, CIN),
                                           smem_desc_kmajor(b_tap + koff, CIN), idesc, k != 0 ? 1u : 0u);
                                }
                        }
                        mma_commit(&tail.acc_full[sl.idx]);
                        mma_commit(&tail.a_empty[st.idx]);   // the stage's Uq is consumed once these MMAs complete
                        st.next(kFStages);
                        sl.next(Cfg::NSLOT);
                    }
            }
            mma_commit(&tail.done);
            mbar_wait_teardown(&tail.done, 0);
        }
    } else {
        // ------------------------------------------------------------ compute warps
        const int cw = warp - 2;                 // 0..7
        const int ctid = threadIdx.x - 64;       // 0..255
        const int quad = warp & 3;               // TMEM lanes 32*quad .. 32*quad+31
        const int half = cw >> 2;                // which 8 of the unit's 16 tiles this warp's epilogue takes
        const int row = 32 * quad + lane;        // output channel of this thread's TMEM lane
        const bool epi = row < COUT;             // uniform per warp (COUT is a multiple of 32)
        const int col0 = 8 * half;
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quad) << 16);
        const int TT = p.TH * p.TW;
        FRing sl{0, 0};
        bool ok = true;
        // the weights' scales, the same for every unit
        for (int i = ctid; i < N2 * NGI * COUT; i += 32 * kFComputeWarps) su_tab[i] = p.sU[i];
        if (epi && lane == 0)
            for (int b = 0; b < Cfg::NSLOT; ++b) mbar_arrive(&tail.acc_empty[b]);   // every slot starts free

        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const long t0 = (long)u * kFNT;
            // ---------------- 1. input transform and quantisation into the operand layout
            for (int i = ctid; i < kFNT * Cfg::NGO; i += 32 * kFComputeWarps) amax[i] = 0u;
#pragma unroll 1
            for (int rnd = 0; rnd < Cfg::ROUNDS; ++rnd) {
                // CIN = 64: a warp is one tile (32 channel pairs); CIN = 32: two tiles of 16 pairs
                const int lt = CIN == 64 ? rnd * kFComputeWarps + cw : 2 * cw + (lane >> 4);
                const int pc = CIN == 64 ? lane : (lane & 15);        // channel pair
                const long t = t0 + lt;
                const bool valid = t < p.T;
                const int img = valid ? (int)(t / TT) : 0;
                const int rem = valid ? (int)(t - (long)img * TT) : 0;
                const int ty = rem / p.TW, tx = rem - (rem / p.TW) * p.TW;
                const Tin* xb = static_cast<const Tin*>(p.x) + (size_t)img * p.H * p.W * CIN + 2 * pc;
                uint64_t v[N][N];
#pragma unroll
                for (int k = 0; k < N; ++k) {
                    const int yy = ty * M - 1 + k;
#pragma unroll
                    for (int l = 0; l < N; ++l) {
                        const int xx = tx * M - 1 + l;
                        v[k][l] = (valid && yy >= 0 && yy < p.H && xx >= 0 && xx < p.W)
                                      ? FPair<Tin>::load(xb + ((size_t)yy * p.W + xx) * CIN)
                                      : 0ull;
                    }
                }
                // T1 = B^T d, in place, column by column
#pragma unroll
                for (int l = 0; l < N; ++l) {
                    uint64_t tcol[N];
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        uint64_t acc = 0ull;
#pragma unroll
                        for (int k = 0; k < N; ++k)
                            if ((MBT >> (i * N + k)) & 1ull) acc = f2_fma(tf.BTd[i * N + k], v[k][l], acc);
                        tcol[i] = acc;
                    }
#pragma unroll
                    for (int i = 0; i < N; ++i) v[i][l] = tcol[i];
                }
                // V = T1 B, in place, row by row
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    uint64_t vrow[N];
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        uint64_t acc = 0ull;
#pragma unroll
                        for (int l = 0; l < N; ++l)
                            if ((MBT >> (j * N + l)) & 1ull) acc = f2_fma(v[i][l], tf.BTd[j * N + l], acc);
                        vrow[j] = acc;
                    }
#pragma unroll
                    for (int j = 0; j < N; ++j) v[i][j] = vrow[j];
                }
                // group maxima per tap in halves of 32 taps, the scales, then the codes
                const int segi = lane / SEG;                 // segment of the warp (SEG = 16: two)
                const int sl_ = lane % SEG;
                const int g = CIN == 64 && G == 32 ? segi : 0;   // input channel group of this lane
                const int col = CIN == 64 ? lt : 2 * cw + segi;  // unit tile of the segment
                float2* qtab = qs_tab + (size_t)(cw * 2 + segi) * 32;
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    if (hb * 32 >= N2) break;
                    float a[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int tap = hb * 32 + e;
                        float lo = 0.0f, hi = 0.0f;
                        if (tap < N2) f2_unpack(v[tap / N][tap % N], lo, hi);
                        a[e] = fmaxf(fabsf(lo), fabsf(hi));
                    }
                    seg_scatter_max32<SEG>(a, lane);
#pragma unroll
                    for (int e = 0; e < 32 / SEG; ++e) {
                        const int te = sl_ * (32 / SEG) + e;      // tap within this half
                        const QScale q = make_qscale(a[e]);
                        qtab[te] = make_float2(q.s, q.r);
                        const int tap = hb * 32 + te;
                        if (tap < N2) {
                            sv[((size_t)tap * NGI + g) * kFNT + col] = q.s;
                            if (DEBUG && valid) p.sV_dbg[((size_t)tap * NGI + g) * p.T_pad + t] = q.s;
                        }
                    }
                    __syncwarp();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int tap = hb * 32 + e;
                        if (tap >= N2) break;
                        const float2 q = qtab[e];
                        const uint32_t codes = quant_pair(v[tap / N][tap % N], q.x, q.y);
                        *reinterpret_cast<uint16_t*>(vq + (size_t)tap * Cfg::VQ_TAP + vq_offset<CIN>(col, 2 * pc)) =
                            (uint16_t)codes;
                        if (DEBUG && valid)
                            *reinterpret_cast<uint16_t*>(p.Vq_dbg + ((size_t)tap * p.T_pad + t) * CIN + 2 * pc) =
                                (uint16_t)codes;
                    }
                    __syncwarp();
                }
            }
            fence_proxy_async_smem();   // the codes are read by the tensor core (async proxy)
            compute_sync();
            if (ctid == 0) mbar_arrive(&tail.vq_ready);

            // ---------------- 2./3. the two GEMM passes
            QScale qy[8];
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                if (pass == 1) {
                    compute_sync();   // every (tile, group) maximum of pass A is in amax
                    if (epi) {
                        const int grp = row / G;
#pragma unroll
                        for (int c = 0; c < 8; ++c) qy[c] = make_qscale(__uint_as_float(amax[(col0 + c) * Cfg::NGO + grp]));
                    }
                }
                if (!epi) continue;
                float mx[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mx[c] = 0.0f;
                for (int s = 0; ok && s < Cfg::NSTEP; ++s) {
                    if (!warp_wait_f(&tail.acc_full[sl.idx], sl.phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t t_slot = t_lane + (uint32_t)(sl.idx * Cfg::SLOT_COLS);
#pragma unroll 1
                    for (int tt = 0; tt < kFTPS; ++tt) {
                        const int tap = s * kFTPS + tt;
                        float y[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) y[c] = 0.0f;
#pragma unroll
                        for (int g = 0; g < NGI; ++g) {
                            uint32_t r[8];
                            tmem_ld<8>(t_slot + (uint32_t)((tt * NGI + g) * kFNT + col0), r);
                            tmem_ld_wait();
                            tmem_regs_ready<8>(r);
                            if (tt + 1 == kFTPS && g + 1 == NGI) {   // the slot is read: release it
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&tail.acc_empty[sl.idx]);
                            }
                            const float su = su_tab[((size_t)tap * NGI + g) * COUT + row];
                            const float4* s4 = reinterpret_cast<const float4*>(sv + ((size_t)tap * NGI + g) * kFNT + col0);
                            const float4 s0 = s4[0], s1 = s4[1];
                            const float svc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                y[c] = __fmaf_rn((float)(int)r[c], __fmul_rn(svc[c], su), y[c]);
                        }
                        if (pass == 0) {
#pragma unroll
                            for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], fabsf(y[c]));
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const int code = quant_one(y[c], qy[c]);
                                yq[((size_t)tap * kFNT + col0 + c) * COUT + row] = (int8_t)code;
                                if (DEBUG && t0 + col0 + c < p.T)
                                    p.Yq_dbg[((size_t)tap * p.T + t0 + col0 + c) * COUT + row] = (int8_t)code;
                            }
                        }
                    }
                    sl.next(Cfg::NSLOT);
                }
                if (pass == 0 && ok) {
                    // maxima over the G output channels of each group: the warp's lanes, then shared memory
                    const int grp = row / G;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float m = mx[c];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) atomicMax(&amax[(col0 + c) * Cfg::NGO + grp], __float_as_uint(m));
                    }
                }
            }
            compute_sync();   // the unit's Yq is complete

            // ---------------- 4. output transform from shared memory
            constexpr int PAIRS = COUT / 2;
#pragma unroll 1
            for (int it = ctid; it < kFNT * PAIRS; it += 32 * kFComputeWarps) {
                const int col = it / PAIRS, co = 2 * (it - col * PAIRS);
                const long t = t0 + col;
                if (t >= p.T) continue;
                const int grp = co / G;
                const float s = group_scale(__uint_as_float(amax[col * Cfg::NGO + grp]));
                if (DEBUG && co % G == 0) p.sY_dbg[(size_t)t * Cfg::NGO + grp] = s;
                const uint64_t s2 = f2_pack(s, s);
                uint64_t Z[M][N];
#pragma unroll
                for (int nu = 0; nu < N; ++nu) {
                    uint64_t Yc[N];
#pragma unroll
                    for (int xi = 0; xi < N; ++xi) {
                        const uint16_t w = *reinterpret_cast<const uint16_t*>(yq + ((size_t)(xi * N + nu) * kFNT + col) * COUT + co);
                        const float q0 = (float)(int8_t)(w & 0xff), q1 = (float)(int8_t)(w >> 8);
                        Yc[xi] = f2_mul(s2, f2_pack(q0, q1));
                    }
#pragma unroll
                    for (int r = 0; r < M; ++r) {
                        uint64_t acc = 0ull;
#pragma unroll
                        for (int xi = 0; xi < N; ++xi)
                            if ((MAT >> (r * N + xi)) & 1ull) acc = f2_fma(tf.ATd[r * N + xi], Yc[xi], acc);
                        Z[r][nu] = acc;
                    }
                }
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
                            if ((MAT >> (c * N + nu)) & 1ull) acc = f2_fma(Z[r][nu], tf.ATd[c * N + nu], acc);
                        float o0, o1;
                        f2_unpack(acc, o0, o1);
                        const size_t o = (((size_t)img * p.H + yy) * p.W + xx) * COUT + co;
                        if (!in_bounds(o + 1, p.n_out, p.err)) continue;
                        if (BF16_OUT)
                            *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p.out) + o) =
                                __floats2bfloat162_rn(o0, o1);
                        else
                            *reinterpret_cast<float2*>(reinterpret_cast<float*>(p.out) + o) = make_float2(o0, o1);
                    }
                }
            }
            // the next unit overwrites Vq, the scales and Yq; all compute warps stop together after an abort
            if (ctid == 0) tail.stop = *abort_flag;
            compute_sync();
            if (tail.stop) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <int M, uint64_t MBT, uint64_t MAT, typename Tin, int CIN, int COUT, int G>
cudaError_t launch_fused_t(const FusedArgs& a, const TransformArgs& tf, int num_sms, cudaStream_t st) {
    using Cfg = FCfg<M, CIN, COUT, G>;
    CUtensorMap tm;
    // Uq [n2][Cout][Cin] int8; box Cin x 128 rows x 4 taps (rows past Cout read zeros), swizzle = Cin bytes
    const cuuint64_t dims[3] = {(cuuint64_t)CIN, (cuuint64_t)COUT, (cuuint64_t)Cfg::N2};
    const cuuint64_t strides[2] = {(cuuint64_t)CIN, (cuuint64_t)COUT * CIN};
    const cuuint32_t box[3] = {(cuuint32_t)CIN, 128u, (cuuint32_t)kFTPS};
    const CUtensorMapSwizzle sw = CIN == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : (CIN == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (!make_tensor_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.Uq, dims, strides, box, sw))
        return cudaErrorInvalidValue;
    const size_t smem = Cfg::BYTES + 1024;
    const long units = (a.T + kFNT - 1) / kFNT;
    const dim3 grid((unsigned)std::min<long>(units, num_sms));
    auto kern = fused_small_kernel<M, MBT, MAT, Tin, CIN, COUT, G>;
    const cudaError_t fe = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (fe != cudaSuccess) return fe;
    return launch_dependent(kern, grid, dim3(kFThreads), smem, st, tm, a, tf);
}

template <int M, uint64_t MBT, uint64_t MAT, typename Tin>
cudaError_t launch_fused_c(const FusedArgs& a, const TransformArgs& tf, int num_sms, cudaStream_t st) {
    if (a.Cin == 64 && a.Cout == 64 && a.G == 32) return launch_fused_t<M, MBT, MAT, Tin, 64, 64, 32>(a, tf, num_sms, st);
    if (a.Cin == 64 && a.Cout == 64 && a.G == 64) return launch_fused_t<M, MBT, MAT, Tin, 64, 64, 64>(a, tf, num_sms, st);
    if (a.Cin == 32 && a.Cout == 32 && a.G == 32) return launch_fused_t<M, MBT, MAT, Tin, 32, 32, 32>(a, tf, num_sms, st);
    return cudaErrorInvalidValue;
}

template <int M, uint64_t MBT, uint64_t MAT>
cudaError_t launch_fused_m(const FusedArgs& a, const TransformArgs& tf, bool bf16_in, int num_sms, cudaStream_t st) {
    return bf16_in ? launch_fused_c<M, MBT, MAT, uint16_t>(a, tf, num_sms, st)
                   : launch_fused_c<M, MBT, MAT, float>(a, tf, num_sms, st);
}

}  // namespace

bool fused_small_fits(int Cin, int Cout, int G) {
    return (Cin == 64 && Cout == 64 && (G == 32 || G == 64)) || (Cin == 32 && Cout == 32 && G == 32);
}

cudaError_t launch_fused_small(const FusedArgs& a, const TransformArgs& tf, int m, bool bf16_in, int num_sms,
                               cudaStream_t st) {
    // the standard point orders (zero-skipping masks of both transforms); the host takes the staged
    // kernels for any other order
    if (m == 2) return launch_fused_m<2, kMaskBT_F2, kMaskAT_F2>(a, tf, bf16_in, num_sms, st);
    if (m == 4) return launch_fused_m<4, kMaskBT_F4, kMaskAT_F4>(a, tf, bf16_in, num_sms, st);
    return launch_fused_m<6, kMaskBT_F6, kMaskAT_F6>(a, tf, bf16_in, num_sms, st);
}

}  // namespace wino
