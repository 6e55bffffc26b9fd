// C ABI of the group-wise fully quantized int8 Winograd convolution library.
// Argument checking, workspace layout and kernel orchestration; all
// arithmetic of the convolution runs in the CUDA kernels.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/wino.h"
#include "kernels.h"
#include "plan.h"

struct wino_plan_s {
    wino::Matrices mat;
    wino::TransformArgs tf;
    wino::WeightArgs wa;
    int G = 0;
    bool bt_masked = false, at_masked = false;
    wino_opts opts;
    int last_cuda = 0;
    // per-kernel timing (wino_profile_begin / wino_profile_end)
    std::vector<cudaEvent_t> prof_events;
    int prof_max_calls = 0, prof_calls = 0, prof_launches = 0;
    // pipelined host entry point: plan-owned copy streams and events on device host_dev
    int host_dev = -1;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    std::vector<cudaEvent_t> host_events;
};

namespace {

using namespace wino;

constexpr size_t kAlign = 256;
size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Guard bands (WINO_DEBUG_GUARDS): kGuardBytes of kGuardByte before every workspace region and
// after the last one, written at the start of each call and checked by wino_check_guards.
constexpr size_t kGuardBytes = 4096;
constexpr unsigned char kGuardByte = 0xA5;
constexpr int kMaxGuards = 12;

struct Layout {
    int TH = 0, TW = 0, n2 = 0, ng = 0, ngo = 0;
    long T = 0, T_pad = 0;
    int y_path = 0, gemm = 0;
    bool dbg_yq = false, dbg_acc = false, ytap = false, xq = false, swap = false, fused = false;
    size_t off_xq = 0, off_vq = 0, off_sv = 0, off_amax = 0, off_yq = 0, off_y32 = 0, off_sy = 0, off_acc = 0, off_err = 0;
    size_t total = 0;
    int n_guards = 0;
    size_t guard[kMaxGuards] = {};
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    }
    return sms;
}

// How Y reaches the output transform when the caller leaves it to the library: the single-pass
// fp32-Y path.  Timed against the two-pass recompute path on every configured layer (ResNet-18/34,
// the SD layers at batch 2 and the 14 shapes of the SD-shaped stack), it is the faster one on each
// (by 6-40 %): the fp32 Y mostly stays in L2 between the GEMM and the output transform, while the
// recompute path reads the operands twice.  The recompute path (a quarter of the Y workspace) runs
// on request.
int auto_y_path() { return WINO_YPATH_Y32; }

int check_shape(const wino_plan_s* p, int N, int H, int W, int Cin, int Cout) {
    if (!p || N <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0) return WINO_ERR_INVALID_ARG;
    if (Cin % p->G != 0 || Cout % p->G != 0 || Cin % 32 != 0 || Cout % 32 != 0) return WINO_ERR_INVALID_ARG;
    return WINO_OK;
}

Layout make_layout(const wino_plan_s* p, int N, int H, int W, int Cin, int Cout) {
    Layout L;
    const int m = p->mat.m, n = p->mat.n;
    L.TH = (H + m - 1) / m;
    L.TW = (W + m - 1) / m;
    L.n2 = n * n;
    L.T = (long)N * L.TH * L.TW;
    L.T_pad = (L.T + 127) / 128 * 128;
    L.ng = Cin / p->G;
    L.ngo = Cout / p->G;
    L.gemm = p->opts.gemm == WINO_GEMM_AUTO ? WINO_GEMM_TCGEN05 : p->opts.gemm;
    if (L.gemm == WINO_GEMM_TCGEN05 && tc_block_n(Cout, p->G) == 0) L.gemm = WINO_GEMM_SIMT;
    L.ytap = p->opts.y_groups == WINO_YGROUPS_TAP;
    // at most 80 tiles: the fp32-Y pass runs with swapped operands (output channels on the MMA's
    // 128 rows), unless the recompute path was asked for
    L.swap = L.gemm == WINO_GEMM_TCGEN05 && tc_swap_ok((int)std::min<long>(L.T, 1 << 30), Cout) &&
             p->opts.y_path != WINO_YPATH_RECOMPUTE;
    L.y_path = (L.ytap || L.swap) ? WINO_YPATH_Y32
                                  : (p->opts.y_path == WINO_YPATH_AUTO ? auto_y_path()
                                                                       : p->opts.y_path);
    L.dbg_yq = (p->opts.debug & WINO_DEBUG_YQ) != 0;
    L.dbg_acc = (p->opts.debug & WINO_DEBUG_ACC32) != 0;
    L.xq = p->opts.x_int8 != 0;
    // the one-kernel path for small channel counts (the recompute path's arithmetic in one launch);
    // on request only: on every configured layer it measures slower than the staged kernels
    L.fused = p->opts.fused == WINO_FUSED_ON && fused_small_fits(Cin, Cout, p->G) && p->bt_masked &&
              p->at_masked && !L.ytap && !L.xq &&
              !L.dbg_acc && p->opts.gemm != WINO_GEMM_SIMT && p->opts.y_path == WINO_YPATH_AUTO &&
              (p->opts.debug & WINO_DEBUG_FORCE_TIMEOUT) == 0;
    if (L.fused) {
        L.y_path = WINO_YPATH_RECOMPUTE;
        L.gemm = WINO_GEMM_TCGEN05;
        L.swap = false;
    }
    const bool guards = (p->opts.debug & WINO_DEBUG_GUARDS) != 0;
    size_t off = 0;
    auto guard = [&]() {
        if (!guards) return;
        L.guard[L.n_guards++] = off;
        off += kGuardBytes;
    };
    if (L.xq) {  // fp32 copy of x after its group-wise int8 round trip
        guard();
        L.off_xq = off;
        off = up(off + sizeof(float) * (size_t)N * H * W * Cin, kAlign);
    }
    // the fused path keeps Vq, its scales and the Y maxima on chip: they exist in the workspace
    // only as its debug copies
    const bool staged = !L.fused || L.dbg_yq;
    if (staged) {
        guard();
        L.off_vq = off;
        off = up(off + (size_t)L.T_pad * L.n2 * Cin, kAlign);
        guard();
        L.off_sv = off;
        off = up(off + sizeof(float) * (size_t)L.n2 * L.ng * L.T_pad, kAlign);
    }
    if (!L.fused) {
        guard();
        L.off_amax = off;
        off = up(off + sizeof(unsigned) * (size_t)L.T_pad * L.ngo, kAlign);
    }
    if ((L.y_path == WINO_YPATH_RECOMPUTE && !L.fused) || L.dbg_yq) {
        guard();
        L.off_yq = off;
        off = up(off + (size_t)L.T * L.n2 * Cout, kAlign);
    }
    if (L.y_path == WINO_YPATH_Y32) {
        guard();
        L.off_y32 = off;
        off = up(off + sizeof(float) * (size_t)L.T * L.n2 * Cout, kAlign);
    }
    if (L.dbg_yq) {
        guard();
        L.off_sy = off;
        off = up(off + sizeof(float) * (size_t)L.T * (L.ytap ? L.n2 : 1) * L.ngo, kAlign);
    }
    if (L.dbg_acc) {
        guard();
        L.off_acc = off;
        off = up(off + sizeof(int) * (size_t)L.n2 * L.T * Cout * L.ng, kAlign);
    }
    guard();
    L.off_err = off;
    off = up(off + 16, kAlign);
    guard();
    L.total = off;
    return L;
}

int cuda_status(wino_plan_s* p, cudaError_t e) {
    if (e == cudaSuccess) return WINO_OK;
    p->last_cuda = (int)e;
    return WINO_ERR_CUDA;
}

constexpr int kMaxHostChunks = 3;

// The last two host calls on each workspace ([0] the latest): their plan, the bytes each one's
// convolution used from the workspace's start (need) and its staging range [lo, hi), and an event
// recorded on its stream when it began (so it fires once every call before it is complete).  The
// next host call on the workspace puts its staging where it touches none of those ranges, when
// that fits, and then orders its input copy only after the older call's event: it streams in
// during both calls' convolutions and output copies.  Any other use of the workspace (the
// device-buffer entry point) ends the chain, and so does destroying a plan of either call.
struct HostCall {
    size_t need = 0, lo = 0, hi = 0;
    cudaEvent_t start = nullptr;
};
struct HostChain {
    const wino_plan_s* plan[2] = {nullptr, nullptr};
    HostCall call[2];
};
std::mutex g_chain_mutex;
std::unordered_map<const void*, HostChain> g_chain;

void chain_erase(std::unordered_map<const void*, HostChain>::iterator it) {
    for (HostCall& c : it->second.call)
        if (c.start) cudaEventDestroy(c.start);
    g_chain.erase(it);
}

void chain_forget_workspace(const void* ws) {
    std::lock_guard<std::mutex> lock(g_chain_mutex);
    auto it = g_chain.find(ws);
    if (it != g_chain.end()) chain_erase(it);
}

void chain_forget_plan(const wino_plan_s* p) {
    std::lock_guard<std::mutex> lock(g_chain_mutex);
    for (auto it = g_chain.begin(); it != g_chain.end();) {
        auto next = std::next(it);
        if (it->second.plan[0] == p || it->second.plan[1] == p) chain_erase(it);
        it = next;
    }
}

// The host entry point's copy streams and events, created on the current device.
int ensure_host_streams(wino_plan_s* p) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(p, e);
    if (p->copy_in && p->host_dev == dev) return WINO_OK;
    for (cudaEvent_t ev : p->host_events) cudaEventDestroy(ev);
    p->host_events.clear();
    if (p->copy_in) cudaStreamDestroy(p->copy_in);
    if (p->copy_out) cudaStreamDestroy(p->copy_out);
    p->copy_in = p->copy_out = nullptr;
    if ((e = cudaStreamCreateWithFlags(&p->copy_in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&p->copy_out, cudaStreamNonBlocking)) != cudaSuccess)
        return cuda_status(p, e);
    p->host_events.assign(1 + 3 * kMaxHostChunks, nullptr);
    for (cudaEvent_t& ev : p->host_events)
        if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_status(p, e);
    p->host_dev = dev;
    return WINO_OK;
}

// Folds a chunk's device error word into the call's (first error wins).
__global__ void error_merge_kernel(int* dst, const int* src) {
    const int v = *src;
    if (v) atomicCAS(dst, 0, v);
}

cudaError_t launch_error_merge(int* dst, const int* src, cudaStream_t st) {
    error_merge_kernel<<<1, 1, 0, st>>>(dst, src);
    return cudaGetLastError();
}

constexpr int kMaxLaunches = 5;

// Records profiling event `slot` of the current call (no-op unless profiling).
void prof_mark(wino_plan_s* p, int slot, cudaStream_t st) {
    if (p->prof_calls >= p->prof_max_calls) return;
    cudaEventRecord(p->prof_events[(size_t)p->prof_calls * (kMaxLaunches + 1) + slot], st);
}

int run_conv(wino_plan_s* p, const void* x, int x_dtype, int N, int H, int W, int Cin, const void* wt, int Cout,
             void* y, int y_dtype, void* ws, size_t ws_bytes, cudaStream_t st) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    if (!x || !wt || !y || !ws || !aligned16(x) || !aligned16(wt) || !aligned16(y) || !aligned16(ws))
        return WINO_ERR_INVALID_ARG;
    if ((x_dtype != WINO_BF16 && x_dtype != WINO_F32) || (y_dtype != WINO_BF16 && y_dtype != WINO_F32))
        return WINO_ERR_INVALID_ARG;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    if (ws_bytes < L.total) return WINO_ERR_WORKSPACE;
    unsigned char* base = static_cast<unsigned char*>(ws);
    int8_t* Vq = reinterpret_cast<int8_t*>(base + L.off_vq);
    float* sV = reinterpret_cast<float*>(base + L.off_sv);
    unsigned* amax = reinterpret_cast<unsigned*>(base + L.off_amax);
    int8_t* Yq = L.off_yq ? reinterpret_cast<int8_t*>(base + L.off_yq) : nullptr;
    float* Y32 = L.off_y32 ? reinterpret_cast<float*>(base + L.off_y32) : nullptr;
    float* sYd = L.dbg_yq ? reinterpret_cast<float*>(base + L.off_sy) : nullptr;
    int* acc = L.dbg_acc ? reinterpret_cast<int*>(base + L.off_acc) : nullptr;
    int* err = reinterpret_cast<int*>(base + L.off_err);
    const int8_t* Uq = static_cast<const int8_t*>(wt);
    const float* sU = reinterpret_cast<const float*>(static_cast<const unsigned char*>(wt) +
                                                     up((size_t)L.n2 * Cout * Cin, kAlign));

    // The error word starts each call at zero.  It is cleared on the stream before the first kernel
    // (not inside a kernel, where the clearing CTA could run after another CTA recorded a timeout).
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
    if (e != cudaSuccess) return cuda_status(p, e);
    for (int gi = 0; gi < L.n_guards; ++gi)
        if ((e = cudaMemsetAsync(base + L.guard[gi], kGuardByte, kGuardBytes, st)) != cudaSuccess)
            return cuda_status(p, e);
    // element counts for the debug build's index checks (one less each under the checks' test hook)
    const size_t sh = (p->opts.debug & WINO_DEBUG_SHRINK_BOUNDS) ? 1 : 0;
    const size_t n_amax = (size_t)L.T_pad * L.ngo - sh, n_y = (size_t)L.T * L.n2 * Cout - sh;
    int slot = 0;
    if (L.fused) {
        FusedArgs fa;
        fa.x = x;
        fa.N = N;
        fa.H = H;
        fa.W = W;
        fa.Cin = Cin;
        fa.Cout = Cout;
        fa.TH = L.TH;
        fa.TW = L.TW;
        fa.G = p->G;
        fa.T = L.T;
        fa.T_pad = L.T_pad;
        fa.Uq = static_cast<const int8_t*>(wt);
        fa.sU = reinterpret_cast<const float*>(static_cast<const unsigned char*>(wt) +
                                               up((size_t)L.n2 * Cout * Cin, kAlign));
        fa.out = y;
        fa.bf16_out = y_dtype == WINO_BF16 ? 1 : 0;
        fa.err = err;
        fa.n_out = (size_t)N * H * W * Cout - sh;
        fa.Vq_dbg = L.dbg_yq ? reinterpret_cast<int8_t*>(base + L.off_vq) : nullptr;
        fa.sV_dbg = L.dbg_yq ? reinterpret_cast<float*>(base + L.off_sv) : nullptr;
        fa.Yq_dbg = L.dbg_yq ? reinterpret_cast<int8_t*>(base + L.off_yq) : nullptr;
        fa.sY_dbg = L.dbg_yq ? reinterpret_cast<float*>(base + L.off_sy) : nullptr;
        prof_mark(p, slot++, st);
        nvtxRangePushA("wino: fused layer");
        e = launch_fused_small(fa, p->tf, p->mat.m, x_dtype == WINO_BF16, num_sms(), st);
        nvtxRangePop();
        prof_mark(p, slot, st);
        if (p->prof_calls < p->prof_max_calls) {
            p->prof_launches = slot;
            ++p->prof_calls;
        }
        return cuda_status(p, e);
    }
    bool x_bf16 = x_dtype == WINO_BF16;
    if (L.xq) {
        float* xq = reinterpret_cast<float*>(base + L.off_xq);
        prof_mark(p, slot++, st);
        nvtxRangePushA("wino: x quantisation");
        e = launch_input_quant(x, x_bf16, (long)N * H * W * Cin, p->G, xq, num_sms(), st);
        nvtxRangePop();
        if (e != cudaSuccess) return cuda_status(p, e);
        x = xq;
        x_bf16 = false;
    }
    InputArgs ia;
    ia.x = x;
    ia.N = N;
    ia.H = H;
    ia.W = W;
    ia.Cin = Cin;
    ia.TH = L.TH;
    ia.TW = L.TW;
    ia.T = L.T;
    ia.T_pad = L.T_pad;
    ia.G = p->G;
    ia.ngo = L.ngo;
    ia.Vq = Vq;
    ia.sV = sV;
    ia.amax = amax;
    ia.err = err;
    ia.num_sms = num_sms();
    ia.n_vq = (size_t)L.T_pad * L.n2 * Cin - sh;
    ia.n_sv = (size_t)L.n2 * L.ng * L.T_pad - sh;
    ia.n_amax = n_amax;
    prof_mark(p, slot++, st);
    nvtxRangePushA("wino: input transform");
    e = launch_input_transform(ia, p->tf, p->mat.m, p->bt_masked, x_bf16, st);
    nvtxRangePop();
    if (e != cudaSuccess) return cuda_status(p, e);

    GemmArgs ga;
    std::memset(&ga, 0, sizeof(ga));
    ga.T = (int)L.T;
    ga.T_pad = (int)L.T_pad;
    ga.Cin = Cin;
    ga.Cout = Cout;
    ga.n2 = L.n2;
    ga.G = p->G;
    ga.ng = L.ng;
    ga.ngo = L.ngo;
    ga.sV = sV;
    ga.sU = sU;
    ga.amax = amax;
    ga.Yq = Yq;
    ga.Y32 = Y32;
    ga.acc = acc;
    ga.err = err;
    ga.force_timeout = (p->opts.debug & WINO_DEBUG_FORCE_TIMEOUT) != 0 && L.gemm == WINO_GEMM_TCGEN05;
    ga.swap_ab = L.swap ? 1 : 0;
    ga.n_v = (size_t)L.T_pad * L.n2 * Cin - sh;
    ga.n_u = (size_t)L.n2 * Cout * Cin - sh;
    ga.n_amax = n_amax;
    ga.n_y = n_y;
    ga.n_acc = (size_t)L.n2 * L.T * Cout * L.ng - sh;
    auto gemm = [&](int mode) -> cudaError_t {
        prof_mark(p, slot++, st);
        nvtxRangePushA(mode == kModeAbsmax ? "wino: hadamard absmax pass"
                                           : (mode == kModeQuant ? "wino: hadamard quantising pass"
                                                                 : "wino: hadamard fp32-Y pass"));
        const cudaError_t ge = L.gemm == WINO_GEMM_SIMT ? launch_hadamard_simt(ga, Vq, Uq, mode, st)
                                                        : launch_hadamard_tc(ga, Vq, Uq, mode, num_sms(), st, nullptr);
        nvtxRangePop();
        return ge;
    };
    if (L.y_path == WINO_YPATH_RECOMPUTE) {
        if ((e = gemm(kModeAbsmax)) != cudaSuccess) return cuda_status(p, e);
        ga.acc = nullptr;
        if ((e = gemm(kModeQuant)) != cudaSuccess) return cuda_status(p, e);
    } else {
        if ((e = gemm(kModeY32)) != cudaSuccess) return cuda_status(p, e);
    }

    OutputArgs oa;
    oa.N = N;
    oa.H = H;
    oa.W = W;
    oa.Cout = Cout;
    oa.TH = L.TH;
    oa.TW = L.TW;
    oa.T = L.T;
    oa.n2 = L.n2;
    oa.G = p->G;
    oa.ngo = L.ngo;
    oa.Yq = Yq;
    oa.Y32 = Y32;
    oa.amax = amax;
    oa.Yq_dbg = (L.y_path == WINO_YPATH_Y32 && L.dbg_yq) ? Yq : nullptr;
    oa.sY_dbg = sYd;
    oa.out = y;
    oa.ytap = L.ytap ? 1 : 0;
    oa.err = err;
    oa.num_sms = num_sms();
    oa.n_y = n_y;
    oa.n_out = (size_t)N * H * W * Cout - sh;
    oa.n_amax = n_amax;
    oa.n_sy = (size_t)L.T * (L.ytap ? L.n2 : 1) * L.ngo - sh;
    prof_mark(p, slot++, st);
    nvtxRangePushA("wino: output transform");
    e = launch_output_transform(oa, p->tf, p->mat.m, p->at_masked, L.y_path == WINO_YPATH_Y32, y_dtype == WINO_BF16,
                                st);
    nvtxRangePop();
    prof_mark(p, slot, st);
    if (p->prof_calls < p->prof_max_calls) {
        p->prof_launches = slot;
        ++p->prof_calls;
    }
    return cuda_status(p, e);
}

}  // namespace

extern "C" {

const char* wino_status_string(int s) {
    switch (s) {
        case WINO_OK: return "ok";
        case WINO_ERR_INVALID_ARG: return "invalid argument";
        case WINO_ERR_UNSUPPORTED: return "unsupported";
        case WINO_ERR_WORKSPACE: return "workspace or weight buffer too small";
        case WINO_ERR_CUDA: return "CUDA error";
        case WINO_ERR_DEVICE_TIMEOUT: return "bounded device wait expired";
        case WINO_ERR_DEVICE_BOUNDS: return "index check failed in a kernel (debug build); the access was skipped";
        case WINO_ERR_GUARD: return "a workspace guard band was overwritten";
        case WINO_ERR_NOT_EXACT: return "transform not exactly representable";
        default: return "unknown status";
    }
}

int wino_plan(wino_plan_t* out, int m, const double* points, const float* S_B, const float* S_G, int group,
              const wino_opts* opts) {
    if (!out) return WINO_ERR_INVALID_ARG;
    *out = nullptr;
    if (group != 32 && group != 64 && group != 256) return WINO_ERR_INVALID_ARG;
    wino_plan_s* p = new (std::nothrow) wino_plan_s();
    if (!p) return WINO_ERR_INVALID_ARG;
    int rc = build_matrices(m, points, S_B, S_G, &p->mat);
    if (rc != WINO_OK) {
        delete p;
        return rc;
    }
    p->G = group;
    std::memset(&p->opts, 0, sizeof(p->opts));
    if (opts) p->opts = *opts;
    if (p->opts.y_path < 0 || p->opts.y_path > 2 || p->opts.gemm < 0 || p->opts.gemm > 2 || p->opts.y_groups < 0 ||
        p->opts.y_groups > 1 || (p->opts.y_groups == WINO_YGROUPS_TAP && p->opts.y_path == WINO_YPATH_RECOMPUTE) ||
        (p->opts.x_int8 != 0 && p->opts.x_int8 != 1) || (p->opts.int8_transforms != 0 && p->opts.int8_transforms != 1) ||
        p->opts.fused < 0 || p->opts.fused > 2) {
        delete p;
        return WINO_ERR_INVALID_ARG;
    }
    if (p->opts.int8_transforms) quantize_transforms_int8(&p->mat);
    const int n = p->mat.n;
    std::memset(&p->tf, 0, sizeof(p->tf));
    std::memcpy(p->tf.BT, p->mat.BT, sizeof(float) * n * n);
    std::memcpy(p->tf.AT, p->mat.AT, sizeof(float) * m * n);
    for (int i = 0; i < n * n; ++i) {
        uint32_t b;
        std::memcpy(&b, &p->mat.BT[i], 4);
        p->tf.BTd[i] = ((uint64_t)b << 32) | b;
    }
    for (int i = 0; i < m * n; ++i) {
        uint32_t b;
        std::memcpy(&b, &p->mat.AT[i], 4);
        p->tf.ATd[i] = ((uint64_t)b << 32) | b;
    }
    std::memcpy(p->wa.G, p->mat.G, sizeof(double) * n * 3);
    const uint64_t bt_mask = m == 2 ? kMaskBT_F2 : (m == 4 ? kMaskBT_F4 : kMaskBT_F6);
    const uint64_t at_mask = m == 2 ? kMaskAT_F2 : (m == 4 ? kMaskAT_F4 : kMaskAT_F6);
    p->bt_masked = (p->mat.bt_nonzero & ~bt_mask) == 0;
    p->at_masked = (p->mat.at_nonzero & ~at_mask) == 0;
    *out = p;
    return WINO_OK;
}

int wino_plan_destroy(wino_plan_t p) {
    if (p) {
        chain_forget_plan(p);
        for (cudaEvent_t ev : p->prof_events) cudaEventDestroy(ev);
        for (cudaEvent_t ev : p->host_events) cudaEventDestroy(ev);
        if (p->copy_in) cudaStreamDestroy(p->copy_in);
        if (p->copy_out) cudaStreamDestroy(p->copy_out);
    }
    delete p;
    return WINO_OK;
}

int wino_plan_matrices(wino_plan_t p, float* BT, double* G, float* AT) {
    if (!p) return WINO_ERR_INVALID_ARG;
    const int m = p->mat.m, n = p->mat.n;
    if (BT) std::memcpy(BT, p->mat.BT, sizeof(float) * n * n);
    if (G) std::memcpy(G, p->mat.G, sizeof(double) * n * 3);
    if (AT) std::memcpy(AT, p->mat.AT, sizeof(float) * m * n);
    return WINO_OK;
}

int wino_plan_info(wino_plan_t p, int* m, int* n, int* group) {
    if (!p) return WINO_ERR_INVALID_ARG;
    if (m) *m = p->mat.m;
    if (n) *n = p->mat.n;
    if (group) *group = p->G;
    return WINO_OK;
}

size_t wino_weight_bytes(wino_plan_t p, int Cin, int Cout) {
    if (!p || Cin <= 0 || Cout <= 0 || Cin % p->G || Cout % p->G) return 0;
    const size_t n2 = (size_t)p->mat.n * p->mat.n;
    return up(n2 * Cout * Cin, kAlign) + up(sizeof(float) * n2 * (Cin / p->G) * Cout, kAlign);
}

int wino_transform_weights(wino_plan_t p, const float* w, int Cin, int Cout, void* wt, size_t wt_bytes, void* stream) {
    if (!p || !w || !wt || !aligned16(w) || !aligned16(wt)) return WINO_ERR_INVALID_ARG;
    if (check_shape(p, 1, 1, 1, Cin, Cout)) return WINO_ERR_INVALID_ARG;
    if (wt_bytes < wino_weight_bytes(p, Cin, Cout)) return WINO_ERR_WORKSPACE;
    const size_t n2 = (size_t)p->mat.n * p->mat.n;
    int8_t* Uq = static_cast<int8_t*>(wt);
    float* sU = reinterpret_cast<float*>(static_cast<unsigned char*>(wt) + up(n2 * Cout * Cin, kAlign));
    return cuda_status(p, launch_weight_transform(p->wa, p->mat.m, w, Cin, Cout, p->G, Uq, sU,
                                                  static_cast<cudaStream_t>(stream)));
}

size_t wino_workspace_bytes(wino_plan_t p, int N, int H, int W, int Cin, int Cout) {
    if (check_shape(p, N, H, W, Cin, Cout)) return 0;
    return make_layout(p, N, H, W, Cin, Cout).total;
}

int wino_conv2d_int8(wino_plan_t p, const void* x, int x_dtype, int N, int H, int W, int Cin, const void* wt,
                      int Cout, void* y, int y_dtype, void* ws, size_t ws_bytes, void* stream) {
    if (!p) return WINO_ERR_INVALID_ARG;
    chain_forget_workspace(ws);
    return run_conv(p, x, x_dtype, N, H, W, Cin, wt, Cout, y, y_dtype, ws, ws_bytes,
                    static_cast<cudaStream_t>(stream));
}

// One call's device staging for x and y.
size_t staging_one(int N, int H, int W, int Cin, int Cout, int x_dtype, int y_dtype) {
    const size_t xs = x_dtype == WINO_BF16 ? 2 : 4, ys = y_dtype == WINO_BF16 ? 2 : 4;
    return up(xs * N * H * W * Cin, kAlign) + up(ys * N * H * W * Cout, kAlign);
}

size_t wino_host_staging_bytes(wino_plan_t p, int N, int H, int W, int Cin, int Cout, int x_dtype, int y_dtype) {
    if (check_shape(p, N, H, W, Cin, Cout)) return 0;
    return 3 * staging_one(N, H, W, Cin, Cout, x_dtype, y_dtype);   // three calls' staging: consecutive calls overlap
}

int wino_conv2d_int8_host(wino_plan_t p, const void* x_host, int x_dtype, int N, int H, int W, int Cin,
                           const void* wt, int Cout, void* y_host, int y_dtype, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!p || !x_host || !y_host || !ws) return WINO_ERR_INVALID_ARG;
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    const size_t need = L.total;
    const size_t stage = staging_one(N, H, W, Cin, Cout, x_dtype, y_dtype);
    if (ws_bytes < need + wino_host_staging_bytes(p, N, H, W, Cin, Cout, x_dtype, y_dtype)) return WINO_ERR_WORKSPACE;
    const size_t xs = x_dtype == WINO_BF16 ? 2 : 4, ys = y_dtype == WINO_BF16 ? 2 : 4;
    const size_t xrow = xs * H * W * Cin, yrow = ys * H * W * Cout;   // bytes per image
    HostChain prev;
    {   // taken out now, set again only when this call is fully enqueued
        std::lock_guard<std::mutex> lock(g_chain_mutex);
        auto it = g_chain.find(ws);
        if (it != g_chain.end()) {
            prev = it->second;
            g_chain.erase(it);   // (its events move to this call's record)
        }
    }
    // Staging: above this call's convolution workspace and, to overlap the last host calls on the
    // workspace (the latest, and the one before it when there is one), above theirs and clear of
    // their staging ranges: the top of the workspace, just below one of their stagings, or right
    // above the highest convolution workspace.  Otherwise right after this call's workspace.
    const int nprev = prev.call[0].start ? (prev.call[1].start ? 2 : 1) : 0;
    size_t s0 = need;
    bool overlap = false;
    if (nprev > 0) {
        size_t floor = need;
        for (int i = 0; i < nprev; ++i) floor = std::max(floor, prev.call[i].need);
        auto clear = [&](size_t a) {
            if (a < floor || a + stage > ws_bytes) return false;
            for (int i = 0; i < nprev; ++i)
                if (a + stage > prev.call[i].lo && a < prev.call[i].hi) return false;
            return true;
        };
        size_t cand[4];
        int nc = 0;
        cand[nc++] = (ws_bytes - stage) / kAlign * kAlign;
        for (int i = 0; i < nprev; ++i)
            if (prev.call[i].lo >= stage) cand[nc++] = (prev.call[i].lo - stage) / kAlign * kAlign;
        cand[nc++] = up(floor, kAlign);
        for (int i = 0; i < nc && !overlap; ++i)
            if (clear(cand[i])) {
                s0 = cand[i];
                overlap = true;
            }
    }
    unsigned char* xd = static_cast<unsigned char*>(ws) + s0;
    unsigned char* yd = xd + up(xrow * N, kAlign);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    // The input copy of an overlapping call waits for the start of the oldest call it overlaps
    // (every call before that one is complete, including the last one to use this staging range).
    cudaEvent_t wait_ev = nprev > 0 ? prev.call[nprev - 1].start : nullptr;
    // This call's start event: the object of the call that drops out of the record (two back),
    // after the wait above has captured its last record, or a new one.
    cudaEvent_t start = nprev == 2 ? prev.call[1].start : nullptr;
    if (!start && (e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming)) != cudaSuccess) {
        if (prev.call[0].start) cudaEventDestroy(prev.call[0].start);   // (the record is dropped)
        return cuda_status(p, e);
    }
    bool recorded = false;   // the start event marks this call on `stream`
    auto finish = [&](int status) {   // record this call as the workspace's latest host call
        std::lock_guard<std::mutex> lock(g_chain_mutex);
        auto it = g_chain.find(ws);
        if (it != g_chain.end()) chain_erase(it);
        HostChain c;
        if (recorded) {
            c.plan[0] = p;
            c.call[0] = HostCall{need, s0, s0 + stage, start};
            c.plan[1] = prev.plan[0];
            c.call[1] = prev.call[0];
        } else {   // (an error before the event was recorded: the next call waits for everything)
            cudaEventDestroy(start);
            if (prev.call[0].start) cudaEventDestroy(prev.call[0].start);
        }
        g_chain[ws] = c;
        return status;
    };

    if (overlap) {
        // The last host calls on this workspace cover this one's input copy: the whole batch is
        // copied in on the copy stream while they compute and copy out, then runs as one
        // convolution on `stream` (its weights read once) and is copied out.
        if ((rc = ensure_host_streams(p)) != WINO_OK) return finish(rc);
        cudaEvent_t* ev = p->host_events.data();
        if ((e = cudaStreamWaitEvent(p->copy_in, wait_ev, 0)) != cudaSuccess) return finish(cuda_status(p, e));
        if ((e = cudaEventRecord(start, st)) != cudaSuccess) return finish(cuda_status(p, e));
        recorded = true;
        if ((e = cudaMemcpyAsync(xd, x_host, xrow * N, cudaMemcpyHostToDevice, p->copy_in)) != cudaSuccess)
            return finish(cuda_status(p, e));
        cudaEventRecord(ev[1], p->copy_in);
        cudaStreamWaitEvent(st, ev[1], 0);
        rc = run_conv(p, xd, x_dtype, N, H, W, Cin, wt, Cout, yd, y_dtype, ws, need, st);
        if (rc) return finish(rc);
        cudaEventRecord(ev[2], st);
        cudaStreamWaitEvent(p->copy_out, ev[2], 0);
        if ((e = cudaMemcpyAsync(y_host, yd, yrow * N, cudaMemcpyDeviceToHost, p->copy_out)) != cudaSuccess)
            return finish(cuda_status(p, e));
        cudaEventRecord(ev[3], p->copy_out);
        return finish(cuda_status(p, cudaStreamWaitEvent(st, ev[3], 0)));
    }

    // Otherwise, chunks of images: every tile, and so every result, belongs to one image, so the
    // chunks give the same bytes as one call.  Two chunk workspaces must fit below the whole
    // call's error word (which collects the chunks' errors).  A chunk's workspace must hold the
    // layout of every chunk size used (the full chunks and the last, smaller one): a smaller chunk
    // can resolve to another kernel variant and need more bytes.
    int K = std::min(N, kMaxHostChunks), Nc = N;
    size_t need_c = need;
    for (; K > 1; --K) {
        Nc = (N + K - 1) / K;
        const int last = N - ((N + Nc - 1) / Nc - 1) * Nc;
        need_c = up(std::max(make_layout(p, Nc, H, W, Cin, Cout).total, make_layout(p, last, H, W, Cin, Cout).total),
                    kAlign);
        if (2 * need_c <= L.off_err) break;
    }
    if (K <= 1) {   // one stream: every step follows all prior work on it
        if ((e = cudaEventRecord(start, st)) != cudaSuccess) return finish(cuda_status(p, e));
        recorded = true;
        if ((e = cudaMemcpyAsync(xd, x_host, xrow * N, cudaMemcpyHostToDevice, st)) != cudaSuccess)
            return finish(cuda_status(p, e));
        rc = run_conv(p, xd, x_dtype, N, H, W, Cin, wt, Cout, yd, y_dtype, ws, need, st);
        if (rc) return finish(rc);
        return finish(cuda_status(p, cudaMemcpyAsync(y_host, yd, yrow * N, cudaMemcpyDeviceToHost, st)));
    }
    K = (N + Nc - 1) / Nc;
    if ((rc = ensure_host_streams(p)) != WINO_OK) return finish(rc);
    cudaEvent_t* ev = p->host_events.data();   // [0]: start, [1 + 3k ..]: in, compute, out of chunk k
    int* err = reinterpret_cast<int*>(static_cast<unsigned char*>(ws) + L.off_err);
    // Without a previous host call to overlap, the input copies wait for all prior work on `stream`
    // (the staging may hold what earlier work still reads); the output copies wait for this call's
    // convolution of their chunk.
    cudaEventRecord(ev[0], st);
    cudaStreamWaitEvent(p->copy_in, ev[0], 0);
    // this call's start on `stream`: the next host call's input copies wait for it
    if ((e = cudaEventRecord(start, st)) != cudaSuccess) return finish(cuda_status(p, e));
    recorded = true;
    if ((e = cudaMemsetAsync(err, 0, sizeof(int), st)) != cudaSuccess) return finish(cuda_status(p, e));
    const unsigned char* xh = static_cast<const unsigned char*>(x_host);
    unsigned char* yh = static_cast<unsigned char*>(y_host);
    for (int k = 0; k < K; ++k) {
        const int n0 = k * Nc, nk = std::min(Nc, N - n0);
        unsigned char* buf = static_cast<unsigned char*>(ws) + (size_t)(k & 1) * need_c;
        if ((e = cudaMemcpyAsync(xd + xrow * n0, xh + xrow * n0, xrow * nk, cudaMemcpyHostToDevice, p->copy_in)) !=
            cudaSuccess)
            return finish(cuda_status(p, e));
        cudaEventRecord(ev[1 + 3 * k], p->copy_in);
        cudaStreamWaitEvent(st, ev[1 + 3 * k], 0);
        rc = run_conv(p, xd + xrow * n0, x_dtype, nk, H, W, Cin, wt, Cout, yd + yrow * n0, y_dtype, buf, need_c, st);
        if (rc) return finish(rc);
        const Layout Lk = make_layout(p, nk, H, W, Cin, Cout);
        if ((e = launch_error_merge(err, reinterpret_cast<const int*>(buf + Lk.off_err), st)) != cudaSuccess)
            return finish(cuda_status(p, e));
        cudaEventRecord(ev[2 + 3 * k], st);
        cudaStreamWaitEvent(p->copy_out, ev[2 + 3 * k], 0);
        if ((e = cudaMemcpyAsync(yh + yrow * n0, yd + yrow * n0, yrow * nk, cudaMemcpyDeviceToHost, p->copy_out)) !=
            cudaSuccess)
            return finish(cuda_status(p, e));
        cudaEventRecord(ev[3 + 3 * k], p->copy_out);
    }
    return finish(cuda_status(p, cudaStreamWaitEvent(st, ev[3 * K], 0)));
}

int wino_check_device_error(wino_plan_t p, const void* ws, int N, int H, int W, int Cin, int Cout, void* stream) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    if (!ws) return WINO_ERR_INVALID_ARG;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(p, e);
    int v = 0;
    e = cudaMemcpy(&v, static_cast<const unsigned char*>(ws) + L.off_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(p, e);
    if (v == 0) return WINO_OK;
    return v == kDevErrBounds ? WINO_ERR_DEVICE_BOUNDS : WINO_ERR_DEVICE_TIMEOUT;
}

int wino_check_guards(wino_plan_t p, const void* ws, int N, int H, int W, int Cin, int Cout, void* stream,
                      int* bad_guard) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    if (!ws) return WINO_ERR_INVALID_ARG;
    if (bad_guard) *bad_guard = -1;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    if (L.n_guards == 0) return WINO_ERR_UNSUPPORTED;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(p, e);
    std::vector<unsigned char> g(kGuardBytes);
    for (int i = 0; i < L.n_guards; ++i) {
        e = cudaMemcpy(g.data(), static_cast<const unsigned char*>(ws) + L.guard[i], kGuardBytes,
                       cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_status(p, e);
        for (unsigned char b : g)
            if (b != kGuardByte) {
                if (bad_guard) *bad_guard = i;
                return WINO_ERR_GUARD;
            }
    }
    return WINO_OK;
}

int wino_debug_dump(wino_plan_t p, const void* ws, int N, int H, int W, int Cin, int Cout, int what, void* dst,
                    size_t bytes) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    if (!ws || !dst) return WINO_ERR_INVALID_ARG;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    const unsigned char* base = static_cast<const unsigned char*>(ws);
    size_t need = 0, off = 0;
    if (L.fused && !L.dbg_yq && (what == WINO_DUMP_VQ || what == WINO_DUMP_SV)) return WINO_ERR_UNSUPPORTED;
    switch (what) {
        case WINO_DUMP_VQ: need = (size_t)L.T * L.n2 * Cin; off = L.off_vq; break;
        case WINO_DUMP_SV: need = sizeof(float) * (size_t)L.T * L.n2 * L.ng; off = L.off_sv; break;
        case WINO_DUMP_YQ:
            if (!L.off_yq || (L.y_path == WINO_YPATH_Y32 && !L.dbg_yq)) return WINO_ERR_UNSUPPORTED;
            need = (size_t)L.T * L.n2 * Cout; off = L.off_yq; break;
        case WINO_DUMP_SY:
            if (!L.dbg_yq) return WINO_ERR_UNSUPPORTED;
            need = sizeof(float) * (size_t)L.T * (L.ytap ? L.n2 : 1) * L.ngo; off = L.off_sy; break;
        case WINO_DUMP_Y32:
            if (!L.off_y32) return WINO_ERR_UNSUPPORTED;
            need = sizeof(float) * (size_t)L.T * L.n2 * Cout; off = L.off_y32; break;
        case WINO_DUMP_ACC32:
            if (!L.dbg_acc) return WINO_ERR_UNSUPPORTED;
            need = sizeof(int) * (size_t)L.n2 * L.T * Cout * L.ng; off = L.off_acc; break;
        default: return WINO_ERR_INVALID_ARG;
    }
    if (bytes < need) return WINO_ERR_WORKSPACE;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(p, e);
    if (what == WINO_DUMP_SY || what == WINO_DUMP_ACC32)
        return cuda_status(p, cudaMemcpy(dst, base + off, need, cudaMemcpyDeviceToHost));
    // The kernels keep these tensors tap-major (Vq [n2][T_pad][Cin]; Yq, Y32 [n2][T][Cout];
    // sV [n2][ng][T_pad]); the dump hands them out tile-major as documented in wino.h.
    size_t esz = 1, inner = 0, rows = 0;  // element size, inner extent, stored rows per tap
    switch (what) {
        case WINO_DUMP_VQ: esz = 1; inner = Cin; rows = L.T_pad; break;
        case WINO_DUMP_SV: esz = 4; inner = L.ng; rows = L.T_pad; break;
        case WINO_DUMP_YQ: esz = 1; inner = Cout; rows = L.T; break;
        default: esz = 4; inner = Cout; rows = L.T; break;  // Y32
    }
    std::vector<unsigned char> raw(esz * inner * rows * L.n2);
    e = cudaMemcpy(raw.data(), base + off, raw.size(), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(p, e);
    unsigned char* o = static_cast<unsigned char*>(dst);
    for (long t = 0; t < L.T; ++t)
        for (int k = 0; k < L.n2; ++k)
            for (size_t c = 0; c < inner; ++c) {
                const size_t src = what == WINO_DUMP_SV ? ((size_t)k * L.ng + c) * L.T_pad + t
                                                        : ((size_t)k * rows + t) * inner + c;
                std::memcpy(o + (((size_t)t * L.n2 + k) * inner + c) * esz, raw.data() + src * esz, esz);
            }
    return WINO_OK;
}

int wino_resolved_config(wino_plan_t p, int N, int H, int W, int Cin, int Cout, int* y_path, int* gemm) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    if (y_path) *y_path = L.y_path;
    if (gemm) *gemm = L.gemm;
    return WINO_OK;
}

int wino_resolved_variants(wino_plan_t p, int N, int H, int W, int Cin, int Cout, int* flags) {
    int rc = check_shape(p, N, H, W, Cin, Cout);
    if (rc) return rc;
    if (!flags) return WINO_ERR_INVALID_ARG;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    int f = 0;
    if (L.fused) {
        *flags = WINO_VARIANT_FUSED;
        return WINO_OK;
    }
    if (L.swap) f |= WINO_VARIANT_SWAPPED_GEMM;
    if (L.gemm == WINO_GEMM_TCGEN05 &&
        tc_a_resident((int)std::min<long>(L.T, 1 << 30), Cin, Cout, p->G, L.swap))
        f |= WINO_VARIANT_A_RESIDENT;
    if (input_transform_split(p->mat.m, p->G, N, L.TH, L.TW, Cin, num_sms())) f |= WINO_VARIANT_SPLIT_INPUT;
    if (output_transform_split(L.T, Cout, L.y_path == WINO_YPATH_Y32, L.ytap, num_sms()))
        f |= WINO_VARIANT_SPLIT_OUTPUT;
    *flags = f;
    return WINO_OK;
}

int wino_launches_per_call(wino_plan_t p, int N, int H, int W, int Cin, int Cout) {
    if (check_shape(p, N, H, W, Cin, Cout)) return 0;
    const Layout L = make_layout(p, N, H, W, Cin, Cout);
    if (L.fused) return 1;
    return (L.y_path == WINO_YPATH_RECOMPUTE ? 4 : 3) + (L.xq ? 1 : 0);
}

int wino_profile_begin(wino_plan_t p, int max_calls) {
    if (!p || max_calls <= 0 || max_calls > (1 << 20)) return WINO_ERR_INVALID_ARG;
    for (cudaEvent_t ev : p->prof_events) cudaEventDestroy(ev);
    p->prof_events.assign((size_t)max_calls * (kMaxLaunches + 1), nullptr);
    for (cudaEvent_t& ev : p->prof_events) {
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) {
            p->prof_max_calls = 0;
            return cuda_status(p, e);
        }
    }
    p->prof_max_calls = max_calls;
    p->prof_calls = 0;
    p->prof_launches = 0;
    return WINO_OK;
}

int wino_profile_end(wino_plan_t p, float* ms, int max_launches, int* launches_per_call, int* calls) {
    if (!p) return WINO_ERR_INVALID_ARG;
    int rc = WINO_OK;
    const int nl = p->prof_launches;
    if (ms)
        for (int i = 0; i < max_launches; ++i) ms[i] = 0.0f;
    if (p->prof_calls > 0) {
        cudaError_t e = cudaEventSynchronize(p->prof_events[(size_t)(p->prof_calls - 1) * (kMaxLaunches + 1) + nl]);
        if (e != cudaSuccess) rc = cuda_status(p, e);
        for (int c = 0; rc == WINO_OK && c < p->prof_calls; ++c)
            for (int i = 0; i < nl && i < max_launches; ++i) {
                float t = 0.0f;
                e = cudaEventElapsedTime(&t, p->prof_events[(size_t)c * (kMaxLaunches + 1) + i],
                                         p->prof_events[(size_t)c * (kMaxLaunches + 1) + i + 1]);
                if (e != cudaSuccess) {
                    rc = cuda_status(p, e);
                    break;
                }
                if (ms) ms[i] += t;
            }
    }
    if (launches_per_call) *launches_per_call = nl;
    if (calls) *calls = p->prof_calls;
    for (cudaEvent_t ev : p->prof_events) cudaEventDestroy(ev);
    p->prof_events.clear();
    p->prof_max_calls = p->prof_calls = p->prof_launches = 0;
    return rc;
}

int wino_last_cuda_error(wino_plan_t p) { return p ? p->last_cuda : 0; }

}  // extern "C"
