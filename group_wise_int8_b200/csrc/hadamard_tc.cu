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
//   stage  = TPS taps x SK bytes of K (SK a multiple of G, so K-groups never
//            straddle stages; TPS > 1 only when one stage holds a tap's whole
//            K); TMA brings the Vq and Uq tiles (3-D boxes over the tap
//            dimension, 32/64/128-byte swizzle) and the sV / sU scales of the
//            stage's groups;
//   warp 0 = TMA producer;
//   warp 1 = TMEM allocator and MMA issuer: tcgen05.mma kind::i8, M=128,
//            N=BN, K=32 per instruction; each K-group of a tap accumulates into
//            its own BN-column TMEM buffer, which holds the int32 bits of
//            1.5*2^23 before the group's first K-step (the epilogue refills it
//            after reading it), so the result reads as that float plus acc; the
//            buffers of one tap form a slot, a ring of at least two slots lets
//            the MMAs run ahead of the epilogue; one wait for a free slot and
//            one commit per tap;
//   warps 2..9 = epilogue, 4 TMEM lane quadrants x 2 column chunks of BN/4:
//            per tap one wait, then per group both chunks' tcgen05.ld, one
//            wait, the buffers refilled with 1.5*2^23 (one tcgen05.st per chunk)
//            and the slot released after its last group, and the
//            dequantisation in packed fp32 pairs, with (float)acc taken
//            exactly as asfloat(0x4B400000 + acc) - 1.5*2^23.  A stage's shared
//            memory returns to the producer when every epilogue warp is done
//            with it (which is after its MMAs completed).
// The loops keep wrap-around ring counters (no division in the issue paths).
// At the end of each tap the epilogue either keeps the running |Y| maximum of
// each (tile, G-cout group) (absmax pass and fp32-Y pass, published with
// atomicMax on the float bits when the CTA leaves a block), writes fp32 Y, or
// requantises Y with sY = absmax/127 and writes int8 Yq.
// Every mbarrier wait is bounded (%globaltimer); on expiry the CTA raises an
// abort flag and the device error word, drains its in-flight TMA loads and
// MMAs, frees its TMEM and returns.
#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

namespace wino {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kMaxStages = 8;
constexpr int kMaxNacc = 8;
constexpr int kMaxKst = 8;         // K stages of a tap kept resident (A-resident walk)
constexpr int kSwapMaxTiles = 80;   // the swapped pass's N is 16, 32 or 80 tiles

template <int BN>
struct TcCfg {
    static constexpr int kCPT = BN / 4;       // columns per column chunk
    static constexpr int kPasses = 2;         // column chunks per epilogue thread
    static constexpr int kEpiWarps = 16 / kPasses;   // 4 TMEM lane quadrants x (4 / kPasses) chunk sets
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kNacc = (512 / BN) < kMaxNacc ? (512 / BN) : kMaxNacc;
    static constexpr int kTmemCols = (kNacc * BN) <= 32 ? 32 : (kNacc * BN) <= 64 ? 64 : (kNacc * BN) <= 128 ? 128
                                     : (kNacc * BN) <= 256 ? 256 : 512;
};

struct SmemTail {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t a_full[kMaxKst];    // A-resident walk: the tap's K stage ks of A has landed
    uint64_t a_empty[kMaxKst];   //   ... and the MMAs of its last column block have read it
    uint64_t acc_full[kMaxNacc];
    uint64_t acc_empty[kMaxNacc];
    uint64_t done;
    uint64_t never;      // completed by nobody: the forced-timeout test hook waits on it
    uint32_t tmem_base;
    int abort_flag;
};

// Ring position with phase bit.
struct Ring {
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

// The tap-units (one tap of one 128-row block and one BN-column block) are
// numbered L = (mb * num_nb + nb) * n2 + tap when there is one column block
// (a stage then covers up to TPS consecutive taps of one block), and
// L = (mb * n2 + tap) * num_nb + nb otherwise (one tap per stage; the column
// blocks of a (row block, tap) follow each other, so its A tile is read from
// DRAM once and the CTAs working on the same taps share the B tiles in L2).
// The units are split into equal contiguous ranges, one per CTA; every role
// of a CTA walks its range the same way, without division.
struct Walk {
    int L, L1, tap, nb, mb;
    __device__ __forceinline__ void init(const GemmArgs& p) {
        const long tot = p.num_units;
        L = (int)(tot * blockIdx.x / gridDim.x);
        L1 = (int)(tot * (blockIdx.x + 1) / gridDim.x);
        if (p.num_nb == 1) {
            tap = L % p.n2;
            nb = 0;
            mb = L / p.n2;
        } else {
            nb = L % p.num_nb;
            const int r = L / p.num_nb;
            tap = r % p.n2;
            mb = r / p.n2;
        }
    }
    __device__ __forceinline__ int stage_taps(int tps, int n2) const { return min(min(tps, n2 - tap), L1 - L); }
    __device__ __forceinline__ void advance(int k, const GemmArgs& p) {
        L += k;
        if (p.num_nb == 1) {
            tap += k;
            if (tap == p.n2) {
                tap = 0;
                ++mb;
            }
        } else {   // k == 1
            if (++nb == p.num_nb) {
                nb = 0;
                if (++tap == p.n2) {
                    tap = 0;
                    ++mb;
                }
            }
        }
    }
};

// Publishes a block's running |Y| maxima into amax [T_pad][Cout/G] (atomicMax on the float bits).
// Rows are tiles: one entry per chunk (its columns lie in one group).  SWAP (rows are output
// channels, columns tiles): per column the maximum over the warp's 32 channels (one group, as
// G >= 32 and a warp's channels start at a multiple of 32), published by lane 0.
template <int NP, int CPT, bool SWAP>
__device__ __forceinline__ void publish_amax(const GemmArgs& p, int row, int lane, const int (&cgrp)[NP],
                                             const int (&colg)[NP], const float (&gmax)[NP],
                                             const float (&gcol)[NP][CPT]) {
#pragma unroll
    for (int h = 0; h < NP; ++h) {
        if (SWAP) {
            const int grp = (row - lane) / p.G;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                float v = gcol[h][c];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                const int tt = colg[h] + c;
                const size_t ai = (size_t)tt * p.ngo + grp;
                if (lane == 0 && tt < p.T && in_bounds(ai, p.n_amax, p.err)) atomicMax(&p.amax[ai], __float_as_uint(v));
            }
        } else {
            const size_t ai = (size_t)row * p.ngo + cgrp[h];
            if (in_bounds(ai, p.n_amax, p.err)) atomicMax(&p.amax[ai], __float_as_uint(gmax[h]));
        }
    }
}

template <int BN, int MODE, bool DUMP, bool SWAP>
__global__ void __launch_bounds__(TcCfg<BN>::kThreads, 1)
    hadamard_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSV, const __grid_constant__ CUtensorMap tmSU, GemmArgs p) {
    using Cfg = TcCfg<BN>;
    constexpr int NACC = Cfg::kNacc;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int BK = p.BK;                   // swizzle width = bytes of K per tile row
    const int KC = p.SK / BK;              // K chunks per stage
    const int TPS = p.tps;                 // taps per stage
    const int GPS = p.SK / p.G;            // K-groups per tap per stage = accumulator buffers per slot
    const int KSTAGES = (p.ng + GPS - 1) / GPS;   // stages per tap (TPS == 1 when > 1); the last may be ragged
    const int GLAST = p.ng - (KSTAGES - 1) * GPS; // K-groups of the last stage (its boxes read zeros past Cin)
    const int NSLOT = NACC / GPS;          // accumulator slots (>= 2)
    const uint32_t a_tile = kBM * BK, b_tile = BN * BK;
    const uint32_t a_bytes = a_tile * KC * TPS, b_bytes = b_tile * KC * TPS;
    // A-resident walk: the tap's KSTAGES A stages first, then a ring of B stages; otherwise a ring
    // of (A, B) stages
    const bool AR = p.a_res != 0;
    const uint32_t a_region = AR ? (uint32_t)KSTAGES * a_bytes : 0u;
    const uint32_t stage_bytes = AR ? b_bytes : a_bytes + b_bytes;   // ring stride
    const uint32_t b_in_stage = AR ? 0u : a_bytes;                   // B's offset within a ring stage
    unsigned char* ring = smem + a_region;
    const int S = p.stages;
    float* sv_ring = reinterpret_cast<float*>(ring + (size_t)S * stage_bytes);   // [S][TPS][GPS][128]
    const int su_stride = (TPS * GPS * BN + 31) / 32 * 32;                         // 128-byte stage slices
    float* su_ring = sv_ring + (size_t)S * TPS * GPS * kBM;                      // [S][su_stride]: [TPS][GPS][BN]
    SmemTail* tail = reinterpret_cast<SmemTail*>(su_ring + (size_t)S * su_stride);
    volatile int* abort_flag = &tail->abort_flag;
    const uint32_t scale_bytes = (uint32_t)TPS * GPS * (kBM + BN) * 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dependents_launch();

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], Cfg::kEpiWarps);   // every epilogue warp, after the stage's MMAs completed
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(&tail->acc_full[b], 1);                 // one commit per tap
            mbar_init(&tail->acc_empty[b], Cfg::kEpiWarps);
        }
        if (AR)
            for (int k = 0; k < KSTAGES; ++k) {
                mbar_init(&tail->a_full[k], 1);
                mbar_init(&tail->a_empty[k], 1);           // one commit after the last column block's MMAs
            }
        mbar_init(&tail->done, 1);
        mbar_init(&tail->never, 1);
        tail->abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSV);
        prefetch_tensormap(&tmSU);
    }
    if (warp == 1) {
        tmem_alloc(&tail->tmem_base, Cfg::kTmemCols);
        tmem_relinquish();
    }
    // barrier setup, TMEM allocation and descriptor prefetch overlap the previous kernel's tail
    grid_dependency_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------- TMA producer
        if (lane == 0) {
            Ring st{0, 0};
            uint32_t issued = 0, pa = 0;   // pa: phase of the resident A stages (one per tap loaded)
            bool ok = true, a_loaded = false, first = true;
            Walk w;
            for (w.init(p); ok && w.L < w.L1;) {
                const int nt = w.stage_taps(TPS, p.n2);
                const bool new_a = AR && (first || w.nb == 0);   // a new (row block, tap): load its A
                first = false;
                for (int ks = 0; ks < KSTAGES; ++ks) {
                    if (new_a) {
                        if (!mbar_wait(&tail->a_empty[ks], pa ^ 1u, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        uint64_t* abar = &tail->a_full[ks];
                        mbar_arrive_expect_tx(abar, a_bytes);
                        for (int c = 0; c < KC; ++c)
                            tma_load_3d(smem + (size_t)ks * a_bytes + (size_t)c * a_tile, &tmA, abar,
                                        ks * p.SK + c * BK, w.mb * kBM, w.tap);
                        a_loaded = true;
                    }
                    if (!mbar_wait(&tail->empty[st.idx], st.phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    // whole boxes of TPS taps; taps past n2 read zeros and taps past the range go unused
                    uint64_t* bar = &tail->full[st.idx];
                    unsigned char* sa = ring + (size_t)st.idx * stage_bytes;
                    mbar_arrive_expect_tx(bar, stage_bytes + scale_bytes);
                    for (int c = 0; c < KC; ++c) {
                        const int k0 = ks * p.SK + c * BK;
                        if (!AR) tma_load_3d(sa + (size_t)c * TPS * a_tile, &tmA, bar, k0, w.mb * kBM, w.tap);
                        tma_load_3d(sa + b_in_stage + (size_t)c * TPS * b_tile, &tmB, bar, k0, w.nb * BN, w.tap);
                    }
                    tma_load_3d(sv_ring + (size_t)st.idx * TPS * GPS * kBM, &tmSV, bar, w.mb * kBM, ks * GPS, w.tap);
                    tma_load_3d(su_ring + (size_t)st.idx * su_stride, &tmSU, bar, w.nb * BN, ks * GPS, w.tap);
                    ++issued;
                    st.next(S);
                }
                if (new_a) pa ^= 1u;
                w.advance(nt, p);
            }
            // drain: every issued load must land before the CTA can exit (the last A stages too)
            if (a_loaded)
                for (int ks = 0; ks < KSTAGES; ++ks) mbar_wait_teardown(&tail->a_full[ks], pa ^ 1u);
            Ring dr{st.idx, st.phase};
            for (uint32_t i = 0; i < issued && i < (uint32_t)S; ++i) {
                if (dr.idx == 0) {
                    dr.idx = S - 1;
                    dr.phase ^= 1u;
                } else {
                    --dr.idx;
                }
                mbar_wait_teardown(&tail->full[dr.idx], dr.phase);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(kBM, BN);
            const uint64_t a_desc0 = smem_desc_kmajor(smem_u32(AR ? smem : ring), BK);
            const uint64_t b_desc0 = smem_desc_kmajor(smem_u32(ring) + b_in_stage, BK);
            const int ks_per_group = p.G / 32;
            const int ks_per_chunk = BK / 32;
            // per K-step of a stage (at most 8: SK <= 256 bytes for G <= 256): the descriptor offsets
            // (16-byte units) of A and B for the stage's first tap and the TMEM column of its K-group,
            // so that a stage's MMAs issue as straight-line code
            uint32_t offa[8], offb[8], dcol[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c = kk / ks_per_chunk, kin = kk - c * ks_per_chunk;
                offa[kk] = (uint32_t)(c * TPS * a_tile + kin * 32) >> 4;
                offb[kk] = (uint32_t)(c * TPS * b_tile + kin * 32) >> 4;
                dcol[kk] = (uint32_t)((kk / ks_per_group) * BN);
            }
            Ring st{0, 0}, sl{0, 0};
            uint32_t pa = 0;
            bool ok = true, first = true;
            if (p.force_timeout) ok = mbar_wait(&tail->never, 0, abort_flag, p.err, 1000000ull);
            Walk w;
            for (w.init(p); ok && w.L < w.L1;) {
                const int nt = w.stage_taps(TPS, p.n2);
                const bool new_a = AR && (first || w.nb == 0);
                const bool last_a = AR && (w.L + 1 == w.L1 || w.nb + 1 == p.num_nb);   // A read for the last time
                first = false;
                for (int ks = 0; ok && ks < KSTAGES; ++ks) {
                    if (new_a && !mbar_wait(&tail->a_full[ks], pa, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&tail->full[st.idx], st.phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint64_t stage_off = (uint64_t)((st.idx * stage_bytes) >> 4);
                    const uint64_t a_off = AR ? (uint64_t)((ks * a_bytes) >> 4) : stage_off;
                    const int ksteps = (ks + 1 == KSTAGES ? GLAST : GPS) * ks_per_group;   // K-steps of this stage
                    for (int t = 0; t < nt; ++t) {
                        if (!mbar_wait(&tail->acc_empty[sl.idx], sl.phase, abort_flag, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + (uint32_t)(sl.idx * GPS * BN);
                        const uint64_t abase = a_desc0 + a_off + (uint64_t)((t * a_tile) >> 4);
                        const uint64_t bbase = b_desc0 + stage_off + (uint64_t)((t * b_tile) >> 4);
                        // every K-step accumulates: the epilogue left the buffer holding the
                        // int32 bits of 1.5*2^23, so it reads asfloat(bits + acc) = 1.5*2^23 + acc
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            if (kk < ksteps) mma_i8(d + dcol[kk], abase + offa[kk], bbase + offb[kk], idesc, 1u);
                        mma_commit(&tail->acc_full[sl.idx]);
                        sl.next(NSLOT);
                    }
                    if (ok && last_a) mma_commit(&tail->a_empty[ks]);   // the A stage is free once these MMAs complete
                    st.next(S);
                }
                if (new_a) pa ^= 1u;
                w.advance(nt, p);
            }
            // all issued MMAs complete before TMEM is released
            mma_commit(&tail->done);
            mbar_wait_teardown(&tail->done, 0);
        }
    } else {
        // ----------------------------------------------------------- epilogue
        // Thread (quad, lane) of epilogue warp ew owns row 32*quad + lane and the
        // column chunks (ew >> 2) + (4 / NP) h, h < NP, of CPT columns each.
        constexpr int CPT = Cfg::kCPT, NP = Cfg::kPasses;
        const int ew = warp - 2;
        const int quad = warp & 3;                    // TMEM lanes 32*quad .. 32*quad+31
        const int rloc = 32 * quad + lane;            // row within the 128-tile block
        int col0[NP];
#pragma unroll
        for (int h = 0; h < NP; ++h) col0[h] = ((ew >> 2) + (4 / NP) * h) * CPT;
        const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quad) << 16);
        // a chunk's fp32 Y row segment starts at a multiple of CPT (8 or 16) floats of a row of Cout (a
        // multiple of 32) floats, so it is 32-byte aligned whenever the Y base is (the workspace
        // itself is only promised 16-byte alignment)
        const bool y32_v8 = CPT % 8 == 0 && (reinterpret_cast<uintptr_t>(p.Y32) & 31u) == 0;
        const uint64_t neg_magic2 = f2_pack(-kRoundMagic, -kRoundMagic);

        // every accumulator buffer starts as the int32 bits of 1.5*2^23 (this warp's lanes and
        // columns), and every slot starts free
        for (int b = 0; b < NSLOT * GPS; ++b)
#pragma unroll
            for (int h = 0; h < NP; ++h) tmem_st_fill<CPT>(t_lane + (uint32_t)(b * BN + col0[h]), (uint32_t)kRoundMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int b = 0; b < NSLOT; ++b) mbar_arrive(&tail->acc_empty[b]);

        Ring st{0, 0}, sl{0, 0};
        bool ok = true;
        int row = 0, blk = -1;
        bool valid = false;
        int colg[NP], cgrp[NP];
        float gmax[NP];
        float gcol[NP][CPT];   // SWAP: running |Y| maximum per column (tile) of this thread's cout
        QScale qy[NP];
#pragma unroll
        for (int h = 0; h < NP; ++h) {
            colg[h] = cgrp[h] = 0;
            gmax[h] = 0.0f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) gcol[h][c] = 0.0f;
            qy[h].s = qy[h].r = 0.0f;
            qy[h].rd = 0.0;
        }
        uint64_t y2[NP][CPT / 2];
        Walk w;
        for (w.init(p); ok && w.L < w.L1;) {
            const int nt = w.stage_taps(TPS, p.n2);
            const int b_id = w.mb * p.num_nb + w.nb;
            if (b_id != blk) {
                // a new (row block, column block): publish the running |Y| maxima of the previous one
                if (MODE != kModeQuant && valid && blk >= 0) publish_amax<NP, CPT, SWAP>(p, row, lane, cgrp, colg, gmax, gcol);
                blk = b_id;
                row = w.mb * kBM + rloc;
                valid = row < (SWAP ? p.Cout : p.T);
#pragma unroll
                for (int h = 0; h < NP; ++h) {
                    colg[h] = w.nb * BN + col0[h];
                    cgrp[h] = colg[h] / p.G;          // CPT <= G: a chunk's columns lie in one Y group
                    gmax[h] = 0.0f;
#pragma unroll
                    for (int c = 0; c < CPT; ++c) gcol[h][c] = 0.0f;
                    const size_t ai = (size_t)row * p.ngo + cgrp[h];
                    if (MODE == kModeQuant && valid && in_bounds(ai, p.n_amax, p.err))
                        qy[h] = make_qscale(__uint_as_float(p.amax[ai]));
                }
            }
            for (int ks = 0; ok && ks < KSTAGES; ++ks) {
                if (!warp_wait(&tail->full[st.idx], st.phase, abort_flag, p.err)) {   // the stage's scales
                    ok = false;
                    break;
                }
                const float* svs = sv_ring + (size_t)st.idx * TPS * GPS * kBM + rloc;
                const float* sus = su_ring + (size_t)st.idx * su_stride;
                for (int t = 0; t < nt; ++t) {
                    const int tap = w.tap + t;
                    if (!warp_wait(&tail->acc_full[sl.idx], sl.phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (ks == 0) {
#pragma unroll
                        for (int h = 0; h < NP; ++h)
#pragma unroll
                            for (int c = 0; c < CPT / 2; ++c) y2[h][c] = 0ull;
                    }
                    const uint32_t t_slot = t_lane + (uint32_t)(sl.idx * GPS * BN);
                    const int gs = ks + 1 == KSTAGES ? GLAST : GPS;   // K-groups of this stage
                    for (int j = 0; j < gs; ++j) {
                        // one group per round, both chunks' loads in flight at once
                        // chunks of more than 16 columns are loaded one at a time (register pressure)
                        constexpr int NR = CPT > 16 ? 1 : NP;
                        uint32_t r[NR][CPT];
                        if constexpr (NR == NP) {
#pragma unroll
                            for (int h = 0; h < NP; ++h) tmem_ld<CPT>(t_slot + (uint32_t)(j * BN + col0[h]), r[h]);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < NP; ++h)   // read: refill for the next accumulation
                                tmem_st_fill<CPT>(t_slot + (uint32_t)(j * BN + col0[h]), (uint32_t)kRoundMagicBits);
                            if (j + 1 == gs) {   // the slot is read and refilled: release it
                                tmem_st_wait();
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&tail->acc_empty[sl.idx]);
                            }
                        }
                        const float sv = svs[(t * GPS + j) * kBM];
                        const uint64_t sv2 = f2_pack(sv, sv);
#pragma unroll
                        for (int h = 0; h < NP; ++h) {
                            const int hr = NR == NP ? h : 0;
                            if constexpr (NR != NP) {
                                tmem_ld<CPT>(t_slot + (uint32_t)(j * BN + col0[h]), r[0]);
                                tmem_ld_wait();
                                tmem_st_fill<CPT>(t_slot + (uint32_t)(j * BN + col0[h]), (uint32_t)kRoundMagicBits);
                                if (h + 1 == NP && j + 1 == gs) {   // the slot is read and refilled: release it
                                    tmem_st_wait();
                                    tc_fence_before();
                                    __syncwarp();
                                    if (lane == 0) mbar_arrive(&tail->acc_empty[sl.idx]);
                                }
                            }
                            const float4* su4 = reinterpret_cast<const float4*>(sus + (t * GPS + j) * BN + col0[h]);
#pragma unroll
                            for (int c4 = 0; c4 < CPT / 4; ++c4) {
                                const float4 uu = su4[c4];
                                // (float)acc exactly: the buffer holds the bits of 1.5*2^23 + acc (|acc| < 2^22)
                                const uint64_t a0 = f2_add(f2_pack(__uint_as_float(r[hr][4 * c4 + 0]),
                                                                   __uint_as_float(r[hr][4 * c4 + 1])),
                                                           neg_magic2);
                                const uint64_t a1 = f2_add(f2_pack(__uint_as_float(r[hr][4 * c4 + 2]),
                                                                   __uint_as_float(r[hr][4 * c4 + 3])),
                                                           neg_magic2);
                                y2[h][2 * c4 + 0] = f2_fma(a0, f2_mul(sv2, f2_pack(uu.x, uu.y)), y2[h][2 * c4 + 0]);
                                y2[h][2 * c4 + 1] = f2_fma(a1, f2_mul(sv2, f2_pack(uu.z, uu.w)), y2[h][2 * c4 + 1]);
                            }
                            if (DUMP && valid) {
                                const int jg = ks * GPS + j;
#pragma unroll
                                for (int c = 0; c < CPT; ++c) {
                                    if (SWAP) {   // row = output channel, column = tile
                                        const size_t di = (((size_t)tap * p.T + colg[h] + c) * p.Cout + row) * p.ng + jg;
                                        if (colg[h] + c < p.T && in_bounds(di, p.n_acc, p.err)) p.acc[di] = (int)(r[hr][c] - kRoundMagicBits);
                                    } else {
                                        const size_t di = (((size_t)tap * p.T + row) * p.Cout + colg[h] + c) * p.ng + jg;
                                        if (in_bounds(di, p.n_acc, p.err)) p.acc[di] = (int)(r[hr][c] - kRoundMagicBits);
                                    }
                                }
                            }
                        }
                    }
                    sl.next(NSLOT);
                    if (ks + 1 < KSTAGES) continue;
                    // ---- end of tap
#pragma unroll
                    for (int h = 0; h < NP; ++h) {
                        float y[CPT];
#pragma unroll
                        for (int c = 0; c < CPT / 2; ++c) f2_unpack(y2[h][c], y[2 * c], y[2 * c + 1]);
                        if constexpr (MODE == kModeQuant) {
                            const size_t yi = ((size_t)tap * p.T + row) * p.Cout + colg[h];
                            if (valid && in_bounds(yi + CPT - 1, p.n_y, p.err)) {
                                uint32_t q[CPT / 4];
                                quant_chunk<CPT>(y, qy[h], q);
                                int8_t* dst = p.Yq + yi;
                                if (CPT == 8) {
                                    *reinterpret_cast<uint2*>(dst) = make_uint2(q[0], q[1 % (CPT / 4)]);
                                } else {
#pragma unroll
                                    for (int c = 0; c < CPT / 16; ++c)
                                        *reinterpret_cast<uint4*>(dst + 16 * c) =
                                            make_uint4(q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
                                }
                            }
                        } else if constexpr (SWAP) {
                            // one output channel, CPT tiles: lanes hold consecutive channels, so each
                            // store instruction writes 32 consecutive floats of one tile and tap
#pragma unroll
                            for (int c = 0; c < CPT; ++c) {
                                const int tt = colg[h] + c;
                                gcol[h][c] = fmaxf(gcol[h][c], fabsf(y[c]));
                                const size_t yi = ((size_t)tap * p.T + tt) * p.Cout + row;
                                if (tt < p.T && in_bounds(yi, p.n_y, p.err)) p.Y32[yi] = y[c];
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < CPT; c += 2) gmax[h] = max_abs3(gmax[h], y[c], y[c + 1]);
                            const size_t yi = ((size_t)tap * p.T + row) * p.Cout + colg[h];
                            if (MODE == kModeY32 && valid && in_bounds(yi + CPT - 1, p.n_y, p.err)) {
                                float* dst = p.Y32 + yi;
                                if (y32_v8) {   // whole 32-byte sectors per store
#pragma unroll
                                    for (int c = 0; c < CPT; c += 8) st_global_v8(dst + c, y + c);
                                } else {
#pragma unroll
                                    for (int c = 0; c < CPT; c += 4)
                                        *reinterpret_cast<float4*>(dst + c) = make_float4(y[c], y[c + 1], y[c + 2], y[c + 3]);
                                }
                            }
                        }
                    }
                }
                // the stage's shared memory (operands read by the completed MMAs, scales read above) is free
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&tail->empty[st.idx]);
                st.next(S);
            }
            w.advance(nt, p);
        }
        if (ok && MODE != kModeQuant && valid && blk >= 0) publish_amax<NP, CPT, SWAP>(p, row, lane, cgrp, colg, gmax, gcol);
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

struct Maps {
    CUtensorMap a, b, sv, su;
};

size_t smem_bytes(const GemmArgs& a, int BN) {
    const size_t gps = (size_t)(a.SK / a.G);
    const size_t kstages = (size_t)((a.ng + (int)gps - 1) / (int)gps);
    const size_t a_region = a.a_res ? kstages * a.SK * kBM : 0;   // the tap's resident A stages
    const size_t per_stage = (size_t)a.tps * a.SK * ((a.a_res ? 0 : kBM) + BN) + (size_t)a.tps * gps * kBM * 4 +
                             ((size_t)a.tps * gps * BN + 31) / 32 * 32 * 4;
    return 1024 + a_region + (size_t)a.stages * per_stage + sizeof(SmemTail);
}

template <int BN, int MODE, bool DUMP, bool SWAP = false>
cudaError_t launch_cfg(const GemmArgs& a, const Maps& m, int num_sms, cudaStream_t st) {
    using Cfg = TcCfg<BN>;
    // at least half the SM's shared memory, so one CTA owns the SM and its TMEM
    const size_t smem = std::max<size_t>(smem_bytes(a, BN), 116 * 1024);
    auto kern = hadamard_tc_kernel<BN, MODE, DUMP, SWAP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = a.num_units < num_sms ? a.num_units : num_sms;   // every CTA gets at least one tap-unit
    return launch_dependent(kern, dim3(grid), dim3(Cfg::kThreads), smem, st, m.a, m.b, m.sv, m.su, a);
}

// Swapped operands: the fp32-Y pass only.
template <int BN>
cudaError_t launch_swap(const GemmArgs& a, const Maps& m, int mode, int num_sms, cudaStream_t st) {
    if (mode != kModeY32) return cudaErrorInvalidValue;
    return a.acc ? launch_cfg<BN, kModeY32, true, true>(a, m, num_sms, st)
                 : launch_cfg<BN, kModeY32, false, true>(a, m, num_sms, st);
}

template <int BN>
cudaError_t launch_bn(const GemmArgs& a, const Maps& m, int mode, int num_sms, cudaStream_t st) {
    const bool dump = a.acc != nullptr && mode != kModeQuant;
    if (mode == kModeAbsmax)
        return dump ? launch_cfg<BN, kModeAbsmax, true>(a, m, num_sms, st)
                    : launch_cfg<BN, kModeAbsmax, false>(a, m, num_sms, st);
    if (mode == kModeQuant) return launch_cfg<BN, kModeQuant, false>(a, m, num_sms, st);
    return dump ? launch_cfg<BN, kModeY32, true>(a, m, num_sms, st) : launch_cfg<BN, kModeY32, false>(a, m, num_sms, st);
}

bool encode(EncodeTiledFn enc, CUtensorMap* map, CUtensorMapDataType dt, const void* base, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
    const cuuint32_t es[3] = {1u, 1u, 1u};
    return enc(map, dt, 3u, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || rank < 1 || rank > 5) return false;
    const cuuint32_t es[5] = {1u, 1u, 1u, 1u, 1u};
    return enc(map, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_block_n(int Cout, int G) {
    if (Cout % 64 == 0) return 64;
    if (Cout % 32 == 0 && G == 32) return 32;
    return 0;
}

// Stage shape: SK bytes of K = GPS K-groups (at most NACC/2, so that at least two accumulator slots
// exist, and at most 256 bytes unless one group is larger); the last stage of a tap holds the
// remaining groups (its boxes past Cin read zeros and its MMAs and epilogue skip them).  Swizzle
// width BK divides SK and G.  TPS taps share a stage when one stage holds a tap's whole K and there
// is one column block (as many as keep three stages in the shared-memory budget).  With several
// column blocks (one tap per stage) a tap's whole A tile stays resident while the CTA walks that
// tap's column blocks, when it fits beside at least three B stages: the A operand then crosses from
// L2 once per (row block, tap) instead of once per column block.
static void choose_stage(GemmArgs& a, int BN) {
    const int nacc = std::min(512 / BN, kMaxNacc);
    const int max_groups = std::max(1, std::min(nacc / 2, std::max(a.G, 256) / a.G));
    const int gps = std::min(max_groups, a.ng);
    const int sk = gps * a.G;
    a.SK = sk;
    a.BK = sk % 128 == 0 ? 128 : (sk % 64 == 0 ? 64 : 32);
    const size_t budget = 200 * 1024;
    const size_t per_tap = (size_t)sk * (kBM + BN) + (size_t)gps * (kBM + BN) * 4;
    a.tps = 1;
    if (sk == a.Cin && a.num_nb == 1)   // several column blocks: one tap per stage (see Walk)
        for (int t : {8, 4, 2})
            if (t <= a.n2 && budget / (per_tap * t) >= 3) {
                a.tps = t;
                break;
            }
    const int kstages = (a.ng + gps - 1) / gps;
    const size_t a_region = (size_t)kstages * sk * kBM;
    const size_t per_b = (size_t)sk * BN + (size_t)gps * (kBM + BN) * 4;
    const size_t ar_budget = 212 * 1024;
    a.a_res = !a.swap_ab && a.num_nb > 1 && a.tps == 1 && kstages <= kMaxKst && a_region < ar_budget &&
              (ar_budget - a_region) / per_b >= 3;
    if (a.a_res) {
        const int stages = (int)((ar_budget - a_region) / per_b);
        a.stages = stages > kMaxStages ? kMaxStages : stages;
        return;
    }
    const int stages = (int)(budget / (per_tap * a.tps));
    a.stages = stages > kMaxStages ? kMaxStages : (stages < 2 ? 2 : stages);
}

bool tc_swap_ok(int T, int Cout) { return T <= kSwapMaxTiles && Cout % kBM == 0; }

bool tc_a_resident(int T, int Cin, int Cout, int G, bool swap) {
    const int BN = swap ? (T <= 16 ? 16 : (T <= 32 ? 32 : 80)) : tc_block_n(Cout, G);
    if (BN == 0 || G <= 0 || Cin % G != 0) return false;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.T = T;
    a.Cin = Cin;
    a.Cout = Cout;
    a.G = G;
    a.ng = Cin / G;
    a.n2 = 64;   // the walk's shape does not depend on the tap count beyond TPS, which is 1 here
    a.swap_ab = swap ? 1 : 0;
    a.num_nb = swap ? (T + BN - 1) / BN : Cout / BN;
    choose_stage(a, BN);
    return a.a_res != 0;
}

cudaError_t launch_hadamard_tc(GemmArgs a, const int8_t* Vq, const int8_t* Uq, int mode, int num_sms,
                               cudaStream_t st, int* launches) {
    const bool swap = a.swap_ab != 0;
    if (swap && (!tc_swap_ok(a.T, a.Cout) || mode != kModeY32)) return cudaErrorInvalidValue;
    // swapped: 128 output channels per row block, the tiles (at most 80) as the MMA's N: 16, 32 or 80
    // (the widths in between spill registers in the epilogue)
    const int BN = swap ? (a.T <= 16 ? 16 : (a.T <= 32 ? 32 : 80)) : tc_block_n(a.Cout, a.G);
    if (BN == 0) return cudaErrorInvalidValue;
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    a.num_mb = swap ? a.Cout / kBM : (a.T + kBM - 1) / kBM;
    a.num_nb = swap ? (a.T + BN - 1) / BN : a.Cout / BN;
    choose_stage(a, BN);
    a.num_units = a.num_mb * a.num_nb * a.n2;   // tap-units, split evenly over the CTAs

    Maps m;
    const CUtensorMapSwizzle sw = swizzle_for(a.BK);
    const int gps = a.SK / a.G;
    // operand A: 128 rows (tiles of Vq, or output channels of Uq when swapped) per row block;
    // operand B: BN rows (output channels of Uq, or tiles of Vq when swapped); the row scales
    // (128 per K-group) and column scales (BN per K-group) follow their operands
    const int8_t* a_src = swap ? Uq : Vq;
    const int8_t* b_src = swap ? Vq : Uq;
    const float* ra_src = swap ? a.sU : a.sV;
    const float* cb_src = swap ? a.sV : a.sU;
    const cuuint64_t rows_v = (cuuint64_t)a.T_pad, rows_u = (cuuint64_t)a.Cout;
    const cuuint64_t a_rows = swap ? rows_u : rows_v, b_rows = swap ? rows_v : rows_u;
    {   // A [n2][a_rows][Cin] int8, box BK x 128 x TPS
        const cuuint64_t dims[3] = {(cuuint64_t)a.Cin, a_rows, (cuuint64_t)a.n2};
        const cuuint64_t strides[2] = {(cuuint64_t)a.Cin, a_rows * a.Cin};
        const cuuint32_t box[3] = {(cuuint32_t)a.BK, (cuuint32_t)kBM, (cuuint32_t)a.tps};
        if (!encode(enc, &m.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_src, dims, strides, box, sw)) return cudaErrorInvalidValue;
    }
    {   // B [n2][b_rows][Cin] int8, box BK x BN x TPS
        const cuuint64_t dims[3] = {(cuuint64_t)a.Cin, b_rows, (cuuint64_t)a.n2};
        const cuuint64_t strides[2] = {(cuuint64_t)a.Cin, b_rows * a.Cin};
        const cuuint32_t box[3] = {(cuuint32_t)a.BK, (cuuint32_t)BN, (cuuint32_t)a.tps};
        if (!encode(enc, &m.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_src, dims, strides, box, sw)) return cudaErrorInvalidValue;
    }
    {   // row scales [n2][ng][a_rows] fp32, box 128 x gps x TPS
        const cuuint64_t dims[3] = {a_rows, (cuuint64_t)a.ng, (cuuint64_t)a.n2};
        const cuuint64_t strides[2] = {a_rows * 4, (cuuint64_t)a.ng * a_rows * 4};
        const cuuint32_t box[3] = {(cuuint32_t)kBM, (cuuint32_t)gps, (cuuint32_t)a.tps};
        if (!encode(enc, &m.sv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ra_src, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    {   // column scales [n2][ng][b_rows] fp32, box BN x gps x TPS
        const cuuint64_t dims[3] = {b_rows, (cuuint64_t)a.ng, (cuuint64_t)a.n2};
        const cuuint64_t strides[2] = {b_rows * 4, (cuuint64_t)a.ng * b_rows * 4};
        const cuuint32_t box[3] = {(cuuint32_t)BN, (cuuint32_t)gps, (cuuint32_t)a.tps};
        if (!encode(enc, &m.su, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cb_src, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (launches) ++*launches;
    if (swap) {
        switch (BN) {
            case 16: return launch_swap<16>(a, m, mode, num_sms, st);
            case 32: return launch_swap<32>(a, m, mode, num_sms, st);
            case 80: return launch_swap<80>(a, m, mode, num_sms, st);
            default: return cudaErrorInvalidValue;
        }
    }
    if (BN == 64) return launch_bn<64>(a, m, mode, num_sms, st);
    return launch_bn<32>(a, m, mode, num_sms, st);
}

}  // namespace wino
