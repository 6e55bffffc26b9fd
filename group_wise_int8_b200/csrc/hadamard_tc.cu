// Hadamard stage on the sm_100a tensor cores ("Data-Free Group-Wise Fully
// Quantized Winograd Convolution via Learnable Scales", Fig. 2: the Hadamard
// product is group-wise quantised; with channels summed it is, per tap, the
// int8 GEMM  Y[tap] = Vq[tap] (T x Cin) . Uq[tap]^T (Cin x Cout)).
//
// Arithmetic (identical to the CUDA-core kernel and the CPU oracle): per
// K-group j of G input channels the tensor core forms the exact int32 dot
// product acc_j; the epilogue computes y = fma((float)acc_j, sV_j * sU_j, y) in
// fp32 for ascending j.
//
// Kernel structure (one CTA per SM, persistent over work units):
//   unit   = (tap chunk, 128-tile row block, BN-cout column block);
//   warp 0 = TMA producer: Vq and Uq K-chunks (BK bytes, 32/64/128-byte
//            swizzle) into a ring of shared-memory stages;
//   warp 1 = TMEM allocator and MMA issuer: tcgen05.mma kind::i8, M=128,
//            N=BN, K=32 per instruction; each K-group accumulates into its own
//            TMEM buffer (a ring of NACC buffers of BN columns) and is
//            committed to an mbarrier when complete;
//   warps 2.. = epilogue: tcgen05.ld of a finished buffer, immediate refill of
//            the buffer with the bias 0x4B400000 (so the next group's int32 sum
//            lands on 1.5*2^23 and reinterprets as an exact fp32 value), then
//            the fp32 dequantisation fma per element.
// At the end of each tap the epilogue either keeps the running |Y| maximum of
// each (tile, G-cout group) (absmax pass and fp32-Y pass, published with
// atomicMax on the float bits at the end of the unit), writes fp32 Y, or
// requantises Y with sY = absmax/127 and writes int8 Yq.
// Every mbarrier wait is bounded (%globaltimer); on expiry the CTA raises an
// abort flag and the device error word, drains its in-flight TMA loads and
// MMAs, frees its TMEM and returns.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace wino {
namespace {

using namespace sm100;

constexpr int kBM = 128;

template <int BN>
struct TcCfg {
    static constexpr int kEpiWarps = BN / 8;        // 4 lane quadrants x BN/32 column chunks
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kCW = BN * 4 / kEpiWarps;  // columns per epilogue thread
    static constexpr int kNacc = (512 / BN) < 8 ? (512 / BN) : 8;
    static constexpr int kTmemCols = (kNacc * BN) <= 32 ? 32 : (kNacc * BN) <= 64 ? 64 : (kNacc * BN) <= 128 ? 128
                                     : (kNacc * BN) <= 256 ? 256 : 512;
};

struct SmemTail {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t acc_full[8];
    uint64_t acc_empty[8];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

// Warp-uniform bounded wait: every lane polls, the loop exits for all lanes together.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
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

__device__ __forceinline__ void decode_unit(const GemmArgs& p, int unit, int& tc, int& mb, int& nb) {
    nb = unit % p.num_nb;
    const int r = unit / p.num_nb;
    mb = r % p.num_mb;
    tc = r / p.num_mb;
}

template <int BN, int MODE, bool DUMP>
__global__ void __launch_bounds__(TcCfg<BN>::kThreads, 1)
    hadamard_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs p) {
    using Cfg = TcCfg<BN>;
    constexpr int CW = Cfg::kCW;
    constexpr int NACC = Cfg::kNacc;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled stage buffers
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int BK = p.BK;
    const int S = p.stages;
    const uint32_t a_bytes = kBM * BK, b_bytes = BN * BK;
    const uint32_t stage_bytes = a_bytes + b_bytes;
    SmemTail* tail = reinterpret_cast<SmemTail*>(smem + (size_t)S * stage_bytes);
    volatile int* abort_flag = &tail->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(&tail->acc_full[b], 1);
            mbar_init(&tail->acc_empty[b], Cfg::kEpiWarps);
        }
        mbar_init(&tail->done, 1);
        tail->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&tail->tmem_base, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int ksteps = p.Cin / 32;        // K-steps of 32 bytes per tap
    const int ks_per_stage = BK / 32;
    const int ks_per_group = p.G / 32;

    if (warp == 0) {
        // ------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t kc = 0;
            bool ok = true;
            for (int unit = blockIdx.x; ok && unit < p.num_units; unit += gridDim.x) {
                int tc, mb, nb;
                decode_unit(p, unit, tc, mb, nb);
                const int tap_end = min(p.n2, (tc + 1) * p.tpu);
                for (int tap = tc * p.tpu; ok && tap < tap_end; ++tap)
                    for (int kb = 0; kb < p.Cin / BK; ++kb) {
                        const int s = kc % S;
                        if (!mbar_wait(&tail->empty[s], ((kc / S) & 1) ^ 1, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        unsigned char* sa = smem + (size_t)s * stage_bytes;
                        mbar_arrive_expect_tx(&tail->full[s], stage_bytes);
                        tma_load_3d(sa, &tmA, &tail->full[s], kb * BK, tap, mb * kBM);
                        tma_load_3d(sa + a_bytes, &tmB, &tail->full[s], kb * BK, nb * BN, tap);
                        ++kc;
                    }
            }
            // drain: every issued load must land before the CTA can exit
            const uint32_t first = kc > (uint32_t)S ? kc - S : 0;
            for (uint32_t i = first; i < kc; ++i) mbar_wait_teardown(&tail->full[i % S], (i / S) & 1);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(kBM, BN);
            uint32_t kc = 0, gc = 0;
            int s = 0, b = 0;
            bool ok = true;
            for (int unit = blockIdx.x; ok && unit < p.num_units; unit += gridDim.x) {
                int tc, mb, nb;
                decode_unit(p, unit, tc, mb, nb);
                const int tap_end = min(p.n2, (tc + 1) * p.tpu);
                for (int tap = tc * p.tpu; ok && tap < tap_end; ++tap)
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const int kin = ks % ks_per_stage;
                        const int gin = ks % ks_per_group;
                        if (kin == 0) {
                            s = kc % S;
                            if (!mbar_wait(&tail->full[s], (kc / S) & 1, abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        if (gin == 0) {
                            b = gc % NACC;
                            if (!mbar_wait(&tail->acc_empty[b], (gc / NACC) & 1, abort_flag, p.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes) + kin * 32;
                        const uint64_t adesc = smem_desc_kmajor(sa, BK);
                        const uint64_t bdesc = smem_desc_kmajor(sa + a_bytes, BK);
                        mma_i8(tmem_base + (uint32_t)(b * BN), adesc, bdesc, idesc, 1u);
                        if (gin == ks_per_group - 1) {
                            mma_commit(&tail->acc_full[b]);
                            ++gc;
                        }
                        if (kin == ks_per_stage - 1) {
                            mma_commit(&tail->empty[s]);
                            ++kc;
                        }
                    }
            }
            // all issued MMAs complete before TMEM is released
            mma_commit(&tail->done);
            mbar_wait_teardown(&tail->done, 0);
        }
    } else {
        // ----------------------------------------------------------- epilogue
        const int ew = warp - 2;
        const int quad = warp & 3;                    // TMEM lanes 32*quad .. 32*quad+31
        const int col0 = (ew / 4) * CW;               // this thread's column chunk in the BN block
        static_assert(CW == 32, "one 32-column TMEM chunk per epilogue thread");
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quad) << 16);
        constexpr int kChunks = CW / 32;              // 32-column chunks; G >= 32, so each lies in one group

        // every accumulator buffer starts filled with the bias
        for (int b = 0; b < NACC; ++b)
#pragma unroll
            for (int cc = 0; cc < CW / 32; ++cc) tmem_st32_fill(t_lane + b * BN + col0 + 32 * cc, (uint32_t)kRoundMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int b = 0; b < NACC; ++b) mbar_arrive(&tail->acc_empty[b]);

        uint32_t gc = 0;
        bool ok = true;
        for (int unit = blockIdx.x; ok && unit < p.num_units; unit += gridDim.x) {
            int tc, mb, nb;
            decode_unit(p, unit, tc, mb, nb);
            const int row = mb * kBM + 32 * quad + lane;
            const bool valid = row < p.T;
            const int colg = nb * BN + col0;
            float gmax[kChunks], sy[kChunks];
#pragma unroll
            for (int k = 0; k < kChunks; ++k) {
                gmax[k] = 0.0f;
                sy[k] = 0.0f;
                if (MODE == kModeQuant && valid)
                    sy[k] = group_scale(__uint_as_float(p.amax[(size_t)row * p.ngo + (colg + 32 * k) / p.G]));
            }
            const int tap_end = min(p.n2, (tc + 1) * p.tpu);
            for (int tap = tc * p.tpu; ok && tap < tap_end; ++tap) {
                float y[CW];
#pragma unroll
                for (int c = 0; c < CW; ++c) y[c] = 0.0f;
                for (int j = 0; j < p.ng; ++j) {
                    const int b = gc % NACC;
                    const float sv = p.sV[((size_t)tap * p.ng + j) * p.T_pad + row];
                    const float* su = p.sU + ((size_t)tap * p.ng + j) * p.Cout + colg;
                    if (!warp_wait(&tail->acc_full[b], (gc / NACC) & 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int cc = 0; cc < kChunks; ++cc) {
                        uint32_t r[32];
                        tmem_ld32(t_lane + b * BN + col0 + 32 * cc, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int c4 = 0; c4 < 32; c4 += 4) {
                            const int c = 32 * cc + c4;
                            const float4 u = __ldg(reinterpret_cast<const float4*>(su + c));
                            y[c + 0] = __fmaf_rn(__fsub_rn(__uint_as_float(r[c4 + 0]), kRoundMagic), __fmul_rn(sv, u.x), y[c + 0]);
                            y[c + 1] = __fmaf_rn(__fsub_rn(__uint_as_float(r[c4 + 1]), kRoundMagic), __fmul_rn(sv, u.y), y[c + 1]);
                            y[c + 2] = __fmaf_rn(__fsub_rn(__uint_as_float(r[c4 + 2]), kRoundMagic), __fmul_rn(sv, u.z), y[c + 2]);
                            y[c + 3] = __fmaf_rn(__fsub_rn(__uint_as_float(r[c4 + 3]), kRoundMagic), __fmul_rn(sv, u.w), y[c + 3]);
                        }
                        if (DUMP && valid) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                p.acc[(((size_t)tap * p.T + row) * p.Cout + colg + 32 * cc + c) * p.ng + j] =
                                    (int)r[c] - kRoundMagicBits;
                        }
                    }
                    // hand the buffer back, refilled with the bias
#pragma unroll
                    for (int cc = 0; cc < kChunks; ++cc)
                        tmem_st32_fill(t_lane + b * BN + col0 + 32 * cc, (uint32_t)kRoundMagicBits);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tail->acc_empty[b]);
                    ++gc;
                }
                if (!ok) break;
                // end of tap
                if (MODE == kModeQuant) {
                    if (valid) {
                        int8_t* dst = p.Yq + ((size_t)row * p.n2 + tap) * p.Cout + colg;
#pragma unroll
                        for (int c = 0; c < CW; c += 16) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                uint32_t pk = 0;
#pragma unroll
                                for (int bb = 0; bb < 4; ++bb) {
                                    const int cc = c + 4 * e + bb;
                                    const int q = quant_code(y[cc], sy[cc / 32]);
                                    pk |= ((uint32_t)(q & 0xff)) << (8 * bb);
                                }
                                w[e] = pk;
                            }
                            *reinterpret_cast<uint4*>(dst + c) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < CW; ++c) gmax[c / 32] = fmaxf(gmax[c / 32], fabsf(y[c]));
                    if (MODE == kModeY32 && valid) {
                        float* dst = p.Y32 + ((size_t)row * p.n2 + tap) * p.Cout + colg;
#pragma unroll
                        for (int c = 0; c < CW; c += 4)
                            *reinterpret_cast<float4*>(dst + c) = make_float4(y[c], y[c + 1], y[c + 2], y[c + 3]);
                    }
                }
            }
            if (ok && MODE != kModeQuant && valid) {
#pragma unroll
                for (int k = 0; k < kChunks; ++k)
                    atomicMax(&p.amax[(size_t)row * p.ngo + (colg + 32 * k) / p.G], __float_as_uint(gmax[k]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

CUtensorMapSwizzle swizzle_for(int bk) {
    return bk == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : (bk == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

template <int BN, int MODE, bool DUMP>
cudaError_t launch_cfg(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, int num_sms, cudaStream_t st) {
    using Cfg = TcCfg<BN>;
    // at least half the SM's shared memory, so one CTA owns the SM and its TMEM
    const size_t smem = std::max<size_t>(1024 + (size_t)a.stages * (kBM + BN) * a.BK + sizeof(SmemTail), 116 * 1024);
    auto kern = hadamard_tc_kernel<BN, MODE, DUMP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = a.num_units < num_sms ? a.num_units : num_sms;
    kern<<<grid, Cfg::kThreads, smem, st>>>(ta, tb, a);
    return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, int mode, int num_sms,
                      cudaStream_t st) {
    const bool dump = a.acc != nullptr && mode != kModeQuant;
    if (mode == kModeAbsmax)
        return dump ? launch_cfg<BN, kModeAbsmax, true>(a, ta, tb, num_sms, st)
                    : launch_cfg<BN, kModeAbsmax, false>(a, ta, tb, num_sms, st);
    if (mode == kModeQuant) return launch_cfg<BN, kModeQuant, false>(a, ta, tb, num_sms, st);
    return dump ? launch_cfg<BN, kModeY32, true>(a, ta, tb, num_sms, st)
                : launch_cfg<BN, kModeY32, false>(a, ta, tb, num_sms, st);
}

}  // namespace

int tc_block_n(int Cout, int G) {
    if (Cout % 128 == 0 && 128 % G == 0) return 128;
    if (Cout % 128 == 0 && G == 256) return 128;
    if (Cout % 64 == 0) return 64;
    if (Cout % 32 == 0 && G == 32) return 32;
    return 0;
}

cudaError_t launch_hadamard_tc(GemmArgs a, const int8_t* Vq, const int8_t* Uq, int mode, int num_sms,
                               cudaStream_t st, int* launches) {
    const int BN = tc_block_n(a.Cout, a.G);
    if (BN == 0) return cudaErrorInvalidValue;
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    a.BK = a.Cin % 128 == 0 ? 128 : (a.Cin % 64 == 0 ? 64 : 32);
    const size_t stage_bytes = (size_t)(kBM + BN) * a.BK;
    int stages = (int)((200 * 1024) / stage_bytes);
    a.stages = stages > 8 ? 8 : (stages < 2 ? 2 : stages);
    a.num_mb = (a.T + kBM - 1) / kBM;
    a.num_nb = a.Cout / BN;
    // tap chunking: enough units to fill the SMs a few times over
    const int base = a.num_mb * a.num_nb;
    int tpu = a.n2;
    while (tpu > 1 && (long)base * ((a.n2 + tpu - 1) / tpu) < 4L * num_sms) tpu = (tpu + 1) / 2;
    a.tpu = tpu;
    a.num_tc = (a.n2 + tpu - 1) / tpu;
    a.num_units = base * a.num_tc;

    CUtensorMap ta, tb;
    {
        cuuint64_t dims[3] = {(cuuint64_t)a.Cin, (cuuint64_t)a.n2, (cuuint64_t)a.T_pad};
        cuuint64_t strides[2] = {(cuuint64_t)a.Cin, (cuuint64_t)a.n2 * a.Cin};
        cuuint32_t box[3] = {(cuuint32_t)a.BK, 1u, (cuuint32_t)kBM};
        cuuint32_t es[3] = {1u, 1u, 1u};
        if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Vq), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(a.BK), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)a.Cin, (cuuint64_t)a.Cout, (cuuint64_t)a.n2};
        cuuint64_t strides[2] = {(cuuint64_t)a.Cin, (cuuint64_t)a.Cout * a.Cin};
        cuuint32_t box[3] = {(cuuint32_t)a.BK, (cuuint32_t)BN, 1u};
        cuuint32_t es[3] = {1u, 1u, 1u};
        if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Uq), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(a.BK), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (launches) ++*launches;
    if (BN == 128) return launch_bn<128>(a, ta, tb, mode, num_sms, st);
    if (BN == 64) return launch_bn<64>(a, ta, tb, mode, num_sms, st);
    return launch_bn<32>(a, ta, tb, mode, num_sms, st);
}

}  // namespace wino
