// Launchers of the Winograd library's CUDA kernels (internal header).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace wino {

// Programmatic dependent launch: every per-call kernel is launched with the
// programmatic stream-serialisation attribute, so its CTAs may be scheduled
// while the previous kernel of the stream drains.  Each such kernel calls
// grid_dependency_wait() before its first global-memory access (it returns once
// the previous grid has completed and its writes are visible) and
// grid_dependents_launch() to let the next kernel be scheduled.  Launched
// without the attribute (or after a kernel that never triggers), both are
// ordinary stream order.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Encodes a tiled TMA tensor map (rank 2..5; strides in bytes for dims 1..rank-1,
// no interleave, no L2 promotion change beyond 256 B, zero fill out of bounds).
bool make_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw);

// ----------------------------------------------------------- weight transform
cudaError_t launch_weight_transform(const WeightArgs& wa, int m, const float* w, int Cin, int Cout, int G,
                                    int8_t* Uq, float* sU, cudaStream_t st);

// ------------------------------------------------------------ input transform
struct InputArgs {
    const void* x;   // [N][H][W][Cin] bf16 or fp32
    int N, H, W, Cin;
    int TH, TW;      // tiles per column / row
    long T;          // N * TH * TW
    long T_pad;      // T rounded up to 128
    int G;
    int ngo;         // Cout / G (rows of the Y absmax table to clear)
    int8_t* Vq;      // [n*n][T_pad][Cin] (tap-major)
    float* sV;       // [n*n][Cin/G][T_pad]
    unsigned* amax;  // [T_pad][Cout/G], cleared here
    int* err;        // device error word (cleared on the stream before the call's first kernel)
    int num_sms;     // SMs of the device (sizes the choice of the split kernel)
    size_t n_vq, n_sv, n_amax;   // element counts of Vq, sV, amax (index checks of the debug build)
};
cudaError_t launch_input_transform(const InputArgs& a, const TransformArgs& tf, int m, bool masked, bool bf16_in,
                                   cudaStream_t st);

// Whether a layer of this shape runs the split input-transform kernel.
bool input_transform_split(int m, int G, int N, int TH, int TW, int Cin, int num_sms);

// Group-wise int8 on x itself: xq = s * Q(x) per G consecutive channels of a pixel
// (elems = N*H*W*Cin values, x bf16 or fp32, xq fp32; both 16-byte aligned).
cudaError_t launch_input_quant(const void* x, bool bf16_in, long elems, int G, float* xq, int num_sms,
                               cudaStream_t st);

// ------------------------------------------------------------ Hadamard GEMM
enum GemmMode { kModeAbsmax = 0, kModeQuant = 1, kModeY32 = 2 };

struct GemmArgs {
    int T, T_pad, Cin, Cout, n2, G, ng, ngo;
    int SK, BK, tps, stages, num_mb, num_nb, num_units;  // stage shape and work split (set by the launcher)
    const float* sV;   // [n2][ng][T_pad]
    const float* sU;   // [n2][ng][Cout]
    unsigned* amax;    // [T_pad][ngo] fp32 bits of |Y| maxima
    int8_t* Yq;        // [n2][T][Cout]   (quant mode)
    float* Y32;        // [n2][T][Cout]   (Y32 mode)
    int* acc;          // [n2][T][Cout][ng] (debug dump) or null
    int* err;
    int force_timeout; // test hook: the MMA thread first waits 1 ms on a barrier nothing completes
    int swap_ab;       // fp32-Y mode, T <= 80, Cout % 128 == 0: the MMA rows are 128 output channels
                       // (A = Uq) and its columns the tiles (B = Vq), so no TMEM lane is padding
    int a_res;         // set by the launcher: a tap's whole A tile stays in shared memory while the
                       // CTA walks that tap's column blocks (several column blocks, one tap per stage)
    size_t n_v, n_u, n_amax, n_y, n_acc;   // element counts of Vq (and sV), Uq (and sU), amax, Yq/Y32 and acc
                                           // (index checks of the debug build)
};

// Tensor maps and launch of the tcgen05 kernel; `Vq` is [n2][T_pad][Cin], `Uq` [n2][Cout][Cin].
cudaError_t launch_hadamard_tc(GemmArgs a, const int8_t* Vq, const int8_t* Uq, int mode, int num_sms,
                               cudaStream_t st, int* launches);
int tc_block_n(int Cout, int G);  // 0 if unsupported
bool tc_swap_ok(int T, int Cout);  // the swapped-operand fp32-Y pass applies (T <= 80, Cout % 128 == 0)
bool tc_a_resident(int T, int Cin, int Cout, int G, bool swap);   // the GEMM keeps a tap's A tile resident

cudaError_t launch_hadamard_simt(const GemmArgs& a, const int8_t* Vq, const int8_t* Uq, int mode, cudaStream_t st);

// --------------------------------------------- fused small-channel layer (x -> out in one kernel)
struct FusedArgs {
    const void* x;            // [N][H][W][Cin] bf16 or fp32
    int N, H, W, Cin, Cout, TH, TW, G;
    long T, T_pad;
    const int8_t* Uq;         // [n2][Cout][Cin]
    const float* sU;          // [n2][Cin/G][Cout]
    void* out;                // [N][H][W][Cout] fp32 or bf16
    int bf16_out;             // 1: bf16 output (round to nearest even), 0: fp32
    int* err;                 // device error word
    size_t n_out;             // elements of out (debug-build index checks)
    int8_t* Vq_dbg;           // debug copies in the staged layouts (or null): Vq [n2][T_pad][Cin],
    float* sV_dbg;            //   sV [n2][Cin/G][T_pad], Yq [n2][T][Cout], sY [T][Cout/G]
    int8_t* Yq_dbg;
    float* sY_dbg;
};
// Whether the fused kernel supports these channel counts and group size (the standard point orders only).
bool fused_small_fits(int Cin, int Cout, int G);
cudaError_t launch_fused_small(const FusedArgs& a, const TransformArgs& tf, int m, bool bf16_in, int num_sms,
                               cudaStream_t st);

// ----------------------------------------------------------- output transform
struct OutputArgs {
    int N, H, W, Cout, TH, TW;
    long T;
    int n2, G, ngo;
    const int8_t* Yq;      // [n2][T][Cout] (Yq source)
    const float* Y32;      // [n2][T][Cout] (Y32 source)
    const unsigned* amax;  // [T_pad][ngo]
    int8_t* Yq_dbg;        // debug copy of Yq (Y32 source), or null
    float* sY_dbg;         // debug copy of sY [T][ngo], or null
    void* out;             // [N][H][W][Cout] fp32 or bf16
    int ytap;              // per-tap Y groups (Y32 source; sY_dbg is then [T][n2][ngo])
    int* err;              // device error word (bounded waits)
    int num_sms;           // SMs of the device (sizes the choice of the split kernel)
    size_t n_y, n_out, n_amax, n_sy;   // element counts of Yq/Y32, out, amax, sY (debug-build index checks)
};
cudaError_t launch_output_transform(const OutputArgs& a, const TransformArgs& tf, int m, bool masked, bool src_y32,
                                    bool bf16_out, cudaStream_t st);
// Whether a layer of this shape runs the split output-transform kernel.
bool output_transform_split(long T, int Cout, bool src_y32, bool ytap, int num_sms);

}  // namespace wino
