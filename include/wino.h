/*
 * wino.h -- C ABI of the B200 (sm_100a) group-wise fully quantized int8
 * Winograd convolution library.
 *
 * The method: "Data-Free Group-Wise Fully Quantized Winograd Convolution via
 * Learnable Scales" (arXiv 2412.19867).  A 3x3, stride-1, pad-1 convolution is
 * computed as F(m,3), m in {4,6}, with transforms built from the Vandermonde
 * factorisation B^T = S_B V^{-T}, G = S_G V, A^T = V^T S_A, S_A = (S_B S_G)^{-1}
 * (review page, "What carries the argument"; Sec. 7.1 "Standard Winograd
 * transforms" for V), and every Winograd stage -- input transform, Hadamard
 * product, output transform -- group-wise quantised to int8 (Fig. 2).
 *
 * Pipeline per call of wino_conv2d_int8 (all stages are CUDA kernels):
 *   input transform   x -> V = B^T d B per tile and channel, int8 Vq with one
 *                     fp32 scale per (tile, tap, G input channels);
 *   Hadamard product  per tap an int8 tensor-core GEMM [tiles x Cin].[Cin x Cout],
 *                     exact int32 per K-group, y = fma(acc_j, sV_j*sU_j, y) in
 *                     fp32, ascending j;
 *   Y requantisation  one fp32 scale per (tile, G output channels) over all
 *                     n*n taps (the cross-shaped per-tap spread of Y, Fig. 3);
 *   output transform  out = A^T (sY Yq) A, cropped, NHWC fp32 or bf16.
 * Quantiser Q everywhere: s = absmax/127, q = clamp(rne(v/s), -127, 127),
 * s = q = 0 for an all-zero group.
 *
 * Conventions
 *  - Status: every function returning int returns WINO_OK (0) or a negative
 *    WINO_ERR_* code.  Nothing aborts, throws or traps; no device trap is used.
 *  - Memory: the caller owns every device buffer and the stream.  The library
 *    owns only the plan (a host object).  Pointers marked _dev are device
 *    pointers, _host are host pointers.  Device pointers must be 16-byte
 *    aligned (WINO_ERR_INVALID_ARG otherwise).
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream).  Launching calls are asynchronous on it; the plan and
 *    query calls are synchronous host calls.
 *  - Layouts: activations NHWC, weights [Cout][3][3][Cin] fp32 (row-major, C
 *    order).  Cin and Cout must be multiples of the group size G.
 *  - Threading: a plan may be used from several host threads as long as the
 *    calls do not share a workspace concurrently.
 */
#ifndef WINO_H_
#define WINO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define WINO_OK 0
#define WINO_ERR_INVALID_ARG (-1)    /* null/misaligned pointer, bad m, G, shape or points */
#define WINO_ERR_UNSUPPORTED (-2)    /* valid request this build does not implement */
#define WINO_ERR_WORKSPACE (-3)      /* workspace or weight buffer smaller than required */
#define WINO_ERR_CUDA (-4)           /* CUDA runtime/driver error; see wino_last_cuda_error */
#define WINO_ERR_DEVICE_TIMEOUT (-5) /* a bounded device wait expired; the kernel returned early */
#define WINO_ERR_NOT_EXACT (-6)      /* transform entries not exactly representable (plan) */
#define WINO_ERR_DEVICE_BOUNDS (-7)  /* debug build: a kernel's index check failed (the access was skipped) */
#define WINO_ERR_GUARD (-8)          /* a workspace guard band was overwritten (WINO_DEBUG_GUARDS) */

/* ----------------------------------------------------------------- dtypes */
#define WINO_F32 0
#define WINO_BF16 1

/* ----------------------------------------------------------------- options */
/* How Y travels from the Hadamard GEMM to the output transform. */
#define WINO_YPATH_AUTO 0      /* the fp32-Y path (measured faster on every configured layer) */
#define WINO_YPATH_RECOMPUTE 1 /* GEMM pass 1: absmax only; pass 2: recompute, quantise, write int8 Yq */
#define WINO_YPATH_Y32 2       /* one GEMM pass writes fp32 Y; the output transform requantises it */

/* Which kernel runs the Hadamard GEMM. */
#define WINO_GEMM_AUTO 0
#define WINO_GEMM_TCGEN05 1 /* TMA + tcgen05.mma kind::i8, TMEM accumulators (default) */
#define WINO_GEMM_SIMT 2    /* CUDA-core integer dot-product kernel, for cross-checks */

typedef struct wino_opts {
    int y_path;    /* WINO_YPATH_* */
    int gemm;      /* WINO_GEMM_* */
    int debug;     /* bit 0: materialise Yq and sY in the workspace on every path;
                      bit 1: dump the int32 per-K-group accumulators (needs the
                             larger workspace wino_workspace_bytes reports);
                      bit 2: failure-detection test hook: the tcgen05 GEMM first
                             waits 1 ms on a barrier nothing completes, so its
                             bounded wait expires, every CTA returns early and
                             wino_check_device_error reports
                             WINO_ERR_DEVICE_TIMEOUT (output undefined);
                      bit 3: guard bands: 4096 bytes of 0xA5 before every
                             workspace region and after the last (the workspace
                             grows accordingly), written at the start of each
                             wino_conv2d_int8 call; wino_check_guards checks them;
                      bit 4: test hook of the debug build's index checks: every
                             element count the kernels check against is one less
                             than its buffer, so the last access of each buffer is
                             skipped and reported as WINO_ERR_DEVICE_BOUNDS (no
                             effect in the release build, which has no checks) */
    int y_groups;  /* WINO_YGROUPS_*: how Y is grouped for its requantisation */
    int x_int8;    /* 0 or 1.  1: group-wise int8 on x itself before the input transform
                      (alternative reading of the input side, Eqs. (14)-(16)): per pixel, G
                      consecutive channels share s = absmax/127 and x becomes
                      s * clamp(rne(x/s), +-127) in fp32; one extra kernel per call, and the
                      workspace holds that fp32 copy of x */
    int int8_transforms; /* 0 or 1.  1: B^T and A^T held as int8 with one scale per matrix
                      (same passage): each entry becomes s * clamp(rne(M/s), +-127) in fp32,
                      s = max|M|/127, at plan time; G stays fp64 (the weights are quantised
                      after their transform) */
    int fused;     /* WINO_FUSED_*: the one-kernel path for small channel counts */
    int reserved;
} wino_opts;

/* The fused path (Cin = Cout = 64 with G = 32 or 64, or Cin = Cout = G = 32; the
 * standard point orders; tile-spanning Y groups, no int8 x, tcgen05 GEMM, automatic Y
 * path, no accumulator dump): one kernel runs the input transform, both GEMM passes of the recompute path
 * and the output transform on units of 16 tiles, with Vq and Yq kept in shared
 * memory; results are identical to the staged kernels.  ON takes it wherever it
 * applies; AUTO and OFF take the staged kernels (on the configured layers the
 * fused kernel is slower: its units of 16 tiles run their phases one after the
 * other, and each stage of 4 taps waits on its own TMA and accumulator
 * handoffs).  With WINO_DEBUG_YQ the
 * kernel also writes Vq, sV, Yq and sY to the workspace for wino_debug_dump. */
#define WINO_FUSED_AUTO 0
#define WINO_FUSED_OFF 1
#define WINO_FUSED_ON 2

/* Y groups (the input of the output transform).  TILE (default, the reading the
 * method needs): one scale per (tile, G consecutive couts) spanning all n*n taps.
 * TAP (alternative reading): one scale per (tile, tap, G couts); it needs the
 * fp32-Y path (y_path AUTO resolves to Y32, RECOMPUTE is rejected) and
 * WINO_DUMP_SY is then [T][n*n][Cout/G]. */
#define WINO_YGROUPS_TILE 0
#define WINO_YGROUPS_TAP 1

#define WINO_DEBUG_YQ 1
#define WINO_DEBUG_ACC32 2
#define WINO_DEBUG_FORCE_TIMEOUT 4
#define WINO_DEBUG_GUARDS 8
#define WINO_DEBUG_SHRINK_BOUNDS 16

/* Debug dump selectors for wino_debug_dump (logical, tile-major layouts of the copy;
 * the kernels keep Vq, sV, Yq and Y tap-major in the workspace). */
#define WINO_DUMP_VQ 0    /* int8  [T][n*n][Cin]        quantised input transform */
#define WINO_DUMP_SV 1    /* fp32  [T][n*n][Cin/G]      its scales */
#define WINO_DUMP_YQ 2    /* int8  [T][n*n][Cout]       requantised Y (needs WINO_DEBUG_YQ on the Y32 path) */
#define WINO_DUMP_SY 3    /* fp32  [T][Cout/G]          Y scales (needs WINO_DEBUG_YQ); [T][n*n][Cout/G] with WINO_YGROUPS_TAP */
#define WINO_DUMP_Y32 4   /* fp32  [T][n*n][Cout]       dequantised Y (Y32 path only) */
#define WINO_DUMP_ACC32 5 /* int32 [n*n][T][Cout][Cin/G] per-K-group accumulators (WINO_DEBUG_ACC32) */

typedef struct wino_plan_s* wino_plan_t;

/*
 * wino_plan -- build the transforms of F(m,3) on the host.
 *   m       2, 4 or 6 (n = m + 2 interpolation points).
 *   points  n doubles, the points in tap order; INFINITY is the point at
 *           infinity (homogeneous (1,0)); finite points must be exact
 *           dyadic-friendly doubles and pairwise distinct.
 *   S_B,S_G n fp32 diagonal scales each, nonzero; NULL = identity.
 *   group   int8 group size G: 32, 64 or 256 (the paper's Sec. 1 sizes).
 *   opts    NULL = defaults (all zero).
 * The Vandermonde inverse is computed in exact rational arithmetic; each
 * entry is rounded once to double, multiplied by the double scale, then
 * rounded to fp32 (B^T, A^T) or kept in double (G).  A^T uses
 * S_A[j] = 1/((double)S_B[j] * (double)S_G[j]).
 * Errors: INVALID_ARG (bad m, group, duplicate or non-finite points, zero
 * scale), NOT_EXACT (a rational does not fit the exact-rounding rule).
 * The plan owns no device memory.  Free with wino_plan_destroy.
 */
int wino_plan(wino_plan_t* out, int m, const double* points, const float* S_B, const float* S_G, int group,
              const wino_opts* opts);
int wino_plan_destroy(wino_plan_t plan);

/* Host copies of the fp32 transforms the kernels use: BT [n][n], AT [m][n]
 * (after int8_transforms, when set), and the fp64 G [n][3] of the weight
 * transform.  Any pointer may be NULL. */
int wino_plan_matrices(wino_plan_t plan, float* BT_host, double* G_host, float* AT_host);

/* m, n, G of a plan; any pointer may be NULL. */
int wino_plan_info(wino_plan_t plan, int* m, int* n, int* group);

/* Bytes of the transformed-weight buffer: int8 Uq [n*n][Cout][Cin] followed
 * (at a 256-byte boundary) by fp32 sU [n*n][Cin/G][Cout].  0 on bad args. */
size_t wino_weight_bytes(wino_plan_t plan, int Cin, int Cout);

/*
 * wino_transform_weights -- offline, once per layer.  U = G g G^T per
 * (cout, cin) in fp64 (fma chains in ascending index from +0), rounded to
 * fp32, then Q over G consecutive input channels at fixed (tap, cout).
 *   w_dev   fp32 [Cout][3][3][Cin] (device).
 *   wt_dev  caller-owned device buffer of wt_bytes >= wino_weight_bytes().
 * Asynchronous on stream.  Errors: INVALID_ARG, WORKSPACE, CUDA.
 */
int wino_transform_weights(wino_plan_t plan, const float* w_dev, int Cin, int Cout, void* wt_dev, size_t wt_bytes,
                           void* stream);

/* Bytes of device workspace wino_conv2d_int8 needs for this shape under the
 * plan's options (includes the debug buffers if the plan enables them). */
size_t wino_workspace_bytes(wino_plan_t plan, int N, int H, int W, int Cin, int Cout);

/*
 * wino_conv2d_int8 -- the hot path: one 3x3 stride-1 pad-1 convolution.
 *   x_dev    [N][H][W][Cin] in x_dtype (WINO_BF16 or WINO_F32), device.
 *   wt_dev   transformed weights from wino_transform_weights (same plan,
 *            Cin, Cout).
 *   y_dev    [N][H][W][Cout] in y_dtype (WINO_F32 or WINO_BF16, RNE), device.
 *   ws_dev   device workspace of ws_bytes >= wino_workspace_bytes().
 * Launches (with x_int8: the quantisation of x, then) the input transform, the
 * Hadamard GEMM (one or two passes) and the output transform on stream.
 * Kernel variants are chosen by shape and give identical bytes: with at most
 * 80 tiles and Cout a multiple of 128, y_path AUTO resolves to Y32 and the GEMM
 * pass runs with swapped operands (output channels on the MMA rows); layers
 * with few tiles per SM run split transform kernels (more threads per tile).
 * The call returns after the launches (asynchronous).
 * A bounded device wait that expires is recorded in the workspace's device
 * error word, and the kernels return early (output undefined).  The call
 * cannot see that itself: call wino_check_device_error on the workspace after
 * the call and before the next call on that workspace, which clears the word
 * (on the stream, before its first kernel).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
int wino_conv2d_int8(wino_plan_t plan, const void* x_dev, int x_dtype, int N, int H, int W, int Cin,
                      const void* wt_dev, int Cout, void* y_dev, int y_dtype, void* ws_dev, size_t ws_bytes,
                      void* stream);

/*
 * wino_conv2d_int8_noalloc -- the same convolution as wino_conv2d_int8 for
 * callers that cannot allocate device memory (no cudaMalloc available or
 * allowed where they run, or no way to pass a workspace through their own
 * interface).  It takes the same inputs and output but no workspace: its
 * scratch is a fixed array of WINO_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.  The
 * call allocates nothing.  (The paper has no counterpart; this is an
 * interface convenience of this library.)
 *   - Shapes whose wino_workspace_bytes() exceeds WINO_NOALLOC_SCRATCH_BYTES
 *     are rejected with WINO_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the array, which keeps the previous call's contents;
 *     the convolution clears what must start at zero itself.  Calls whose
 *     kernels overlap on the GPU race on the array: order them.
 *   - A bounded device wait that expires is recorded in the array's device
 *     error word: call wino_check_device_error_noalloc after the call and
 *     before the next call, which clears the word.
 * Errors: INVALID_ARG, WORKSPACE, CUDA, plus those of wino_conv2d_int8.
 */
#define WINO_NOALLOC_SCRATCH_BYTES (64u << 20)
int wino_conv2d_int8_noalloc(wino_plan_t plan, const void* x_dev, int x_dtype, int N, int H, int W, int Cin,
                             const void* wt_dev, int Cout, void* y_dev, int y_dtype, void* stream);

/* wino_check_device_error for wino_conv2d_int8_noalloc: synchronises stream and
 * reads the device error word the last call of this shape and plan left in the
 * library's scratch array: WINO_OK, or WINO_ERR_DEVICE_TIMEOUT if a bounded wait
 * in a kernel expired.  (No counterpart in the paper.)  Errors: INVALID_ARG,
 * WORKSPACE (shape beyond the array), CUDA. */
int wino_check_device_error_noalloc(wino_plan_t plan, int N, int H, int W, int Cin, int Cout, void* stream);

/* Extra device bytes wino_conv2d_int8_host needs beyond wino_workspace_bytes:
 * device staging for x and y, three times (room for three calls' staging, so
 * that consecutive host calls on one workspace overlap; see below). */
size_t wino_host_staging_bytes(wino_plan_t plan, int N, int H, int W, int Cin, int Cout, int x_dtype,
                               int y_dtype);

/*
 * wino_conv2d_int8_host -- same convolution with HOST input and output
 * buffers: copies x_host to the device, runs the convolution, copies the
 * result to y_host, all asynchronously with respect to stream (pinned host
 * memory gives truly asynchronous copies).  When N >= 2 the batch is cut into
 * up to 3 chunks of images, pipelined: the copy of chunk k+1 in and of chunk
 * k-1 out overlap the convolution of chunk k (the copies run on two streams
 * the plan owns, ordered after and before `stream` by events; results are
 * identical to one call, every tile belonging to one image).  ws_dev must hold
 * wino_workspace_bytes() + wino_host_staging_bytes() (else WINO_ERR_WORKSPACE).
 * The caller synchronises `stream` before reading y_host.  Calls on one plan
 * must not run concurrently.  Consecutive host calls on one workspace (any
 * plans and shapes, issued on one stream) overlap: a call stages x and y where
 * they touch neither the last two host calls' convolution workspaces nor their
 * staging (the top of ws_dev, just below one of their stagings, or above the
 * largest of the three convolution workspaces), its input copy then waits only
 * until every call before those two is complete, so it streams in during their
 * convolutions and output copies, and the batch runs as one convolution (its
 * weights read once).  When no such
 * place fits in ws_bytes (a workspace sized for a
 * smaller shape), the call waits for all prior work on `stream`, and so does
 * the first host call after a wino_conv2d_int8 call on ws_dev.  Work outside
 * this library must not use ws_dev, and x_host must not change until the
 * call's work on `stream` has completed.
 */
int wino_conv2d_int8_host(wino_plan_t plan, const void* x_host, int x_dtype, int N, int H, int W, int Cin,
                           const void* wt_dev, int Cout, void* y_host, int y_dtype, void* ws_dev, size_t ws_bytes,
                           void* stream);

/* Synchronises stream and reads the workspace's device error word left by the
 * last call on ws_dev: WINO_OK, WINO_ERR_DEVICE_TIMEOUT if a bounded wait in a
 * kernel expired, or (debug build only, libwino_b200_debug.so, compiled with
 * WINO_DEBUG) WINO_ERR_DEVICE_BOUNDS if a kernel's index check found an
 * element index outside its buffer and skipped the access.  The next call on
 * the workspace clears the word, so check between calls. */
int wino_check_device_error(wino_plan_t plan, const void* ws_dev, int N, int H, int W, int Cin, int Cout,
                            void* stream);

/* Guard bands (plan option WINO_DEBUG_GUARDS): synchronises stream and checks
 * that every guard band of the workspace layout of this shape still holds its
 * pattern after the last wino_conv2d_int8 call on ws_dev.  Returns WINO_OK, or
 * WINO_ERR_GUARD with *bad_guard (may be NULL) set to the index of the first
 * overwritten band in layout order; WINO_ERR_UNSUPPORTED if the plan has no
 * guard bands.  (A stand-in for a memory checker, which is not available where
 * this library is tested; no counterpart in the paper.) */
int wino_check_guards(wino_plan_t plan, const void* ws_dev, int N, int H, int W, int Cin, int Cout, void* stream,
                      int* bad_guard);

/* Synchronous copy of one intermediate tensor of the last call on ws_dev
 * into host_dst (logical layout per WINO_DUMP_*).  Errors: INVALID_ARG,
 * UNSUPPORTED (tensor not materialised under these options), WORKSPACE. */
int wino_debug_dump(wino_plan_t plan, const void* ws_dev, int N, int H, int W, int Cin, int Cout, int what,
                    void* host_dst, size_t host_bytes);

/* The Y path and GEMM kernel a call of this shape will use (after AUTO). */
int wino_resolved_config(wino_plan_t plan, int N, int H, int W, int Cin, int Cout, int* y_path, int* gemm);

/* Kernel variants a call of this shape runs (all give the same bytes), as a
 * bit set of WINO_VARIANT_*: the swapped-operand GEMM pass, the split input
 * and output transforms (more threads per tile; sized by the device's SM count,
 * 148 assumed when no device is visible), the fused small-channel kernel, and
 * the GEMM walk that keeps a tap's A tile resident in shared memory across its
 * column blocks.  Errors: INVALID_ARG. */
#define WINO_VARIANT_SWAPPED_GEMM 1
#define WINO_VARIANT_SPLIT_INPUT 2
#define WINO_VARIANT_SPLIT_OUTPUT 4
#define WINO_VARIANT_FUSED 8
#define WINO_VARIANT_A_RESIDENT 16
int wino_resolved_variants(wino_plan_t plan, int N, int H, int W, int Cin, int Cout, int* flags);

/* Number of kernels one wino_conv2d_int8 call of this shape launches. */
int wino_launches_per_call(wino_plan_t plan, int N, int H, int W, int Cin, int Cout);

/*
 * Per-kernel device timing.  wino_profile_begin(plan, max_calls) makes the
 * next max_calls calls of wino_conv2d_int8 on this plan record a CUDA event on
 * their stream before each kernel launch and after the last one (the events
 * are owned by the plan).  wino_profile_end synchronises on the last event
 * and returns, per launch index (input transform, GEMM pass(es), output
 * transform), the summed elapsed milliseconds over the recorded calls, the
 * number of launches per call and the number of calls recorded; it then
 * releases the events.  Errors: INVALID_ARG, CUDA.
 */
int wino_profile_begin(wino_plan_t plan, int max_calls);
int wino_profile_end(wino_plan_t plan, float* ms_per_launch, int max_launches, int* launches_per_call,
                     int* calls);

/* Last CUDA error code seen by this plan (cudaError_t as int), 0 if none. */
int wino_last_cuda_error(wino_plan_t plan);

/* Static description of a status code. */
const char* wino_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* WINO_H_ */
