// Hadamard stage on CUDA cores (cross-check kernel for the tensor-core one).
// Per tap, tile and output channel: acc_j = exact int32 dot product of the
// G int8 pairs of K-group j (dp4a), y = fma((float)acc_j, sV_j * sU_j, y) in
// fp32 for ascending j -- the same arithmetic as the tcgen05 kernel, one
// thread per output.  Epilogue modes as in the tcgen05 kernel: Y absmax
// (per tile and G-cout group, over taps, via atomicMax on the float bits),
// requantisation to int8 with sY = absmax/127, or fp32 Y.
#include "kernels.h"

namespace wino {
namespace {

template <int MODE, bool DUMP>
__global__ void __launch_bounds__(256) hadamard_simt_kernel(GemmArgs p, const int8_t* __restrict__ Vq,
                                                            const int8_t* __restrict__ Uq) {
    grid_dependents_launch();
    grid_dependency_wait();
    const int tap = blockIdx.y;
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long t = i / p.Cout;
    const int co = (int)(i - t * p.Cout);
    if (t >= p.T) return;  // Cout % 32 == 0: uniform per warp
    const size_t vrow = ((size_t)tap * p.T_pad + t) * p.Cin, urow = ((size_t)tap * p.Cout + co) * p.Cin;
    if (!in_bounds(vrow + p.Cin - 1, p.n_v, p.err) || !in_bounds(urow + p.Cin - 1, p.n_u, p.err)) return;
    const int4* v = reinterpret_cast<const int4*>(Vq + ((size_t)tap * p.T_pad + t) * p.Cin);
    const int4* u = reinterpret_cast<const int4*>(Uq + ((size_t)tap * p.Cout + co) * p.Cin);
    float y = 0.0f;
    for (int j = 0; j < p.ng; ++j) {
        int acc = 0;
        for (int c = 0; c < p.G / 16; ++c) {
            const int4 a = v[j * (p.G / 16) + c], b = __ldg(&u[j * (p.G / 16) + c]);
            acc = __dp4a(a.x, b.x, acc);
            acc = __dp4a(a.y, b.y, acc);
            acc = __dp4a(a.z, b.z, acc);
            acc = __dp4a(a.w, b.w, acc);
        }
        const size_t di = (((size_t)tap * p.T + t) * p.Cout + co) * p.ng + j;
        if (DUMP && in_bounds(di, p.n_acc, p.err)) p.acc[di] = acc;
        const float pr = __fmul_rn(p.sV[((size_t)tap * p.ng + j) * p.T_pad + t], p.sU[((size_t)tap * p.ng + j) * p.Cout + co]);
        y = __fmaf_rn((float)acc, pr, y);
    }
    const size_t o = ((size_t)tap * p.T + t) * p.Cout + co;
    const size_t ai = (size_t)t * p.ngo + co / p.G;
    if (!in_bounds(o, p.n_y, p.err) || !in_bounds(ai, p.n_amax, p.err)) return;
    unsigned* am = p.amax + ai;
    if (MODE == kModeQuant) {
        p.Yq[o] = (int8_t)quant_code(y, group_scale(__uint_as_float(*am)));
    } else {
        if (MODE == kModeY32) p.Y32[o] = y;
        const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(y)));
        if ((threadIdx.x & 31) == 0) atomicMax(am, m);  // a warp's 32 couts lie in one group (G >= 32)
    }
}

}  // namespace

cudaError_t launch_hadamard_simt(const GemmArgs& a, const int8_t* Vq, const int8_t* Uq, int mode, cudaStream_t st) {
    const long threads = (long)a.T * a.Cout;
    const dim3 grid((unsigned)((threads + 255) / 256), a.n2);
    const bool dump = a.acc != nullptr && mode != kModeQuant;
    if (mode == kModeAbsmax)
        return dump ? launch_dependent(hadamard_simt_kernel<kModeAbsmax, true>, grid, dim3(256), 0, st, a, Vq, Uq)
                    : launch_dependent(hadamard_simt_kernel<kModeAbsmax, false>, grid, dim3(256), 0, st, a, Vq, Uq);
    if (mode == kModeQuant)
        return launch_dependent(hadamard_simt_kernel<kModeQuant, false>, grid, dim3(256), 0, st, a, Vq, Uq);
    return dump ? launch_dependent(hadamard_simt_kernel<kModeY32, true>, grid, dim3(256), 0, st, a, Vq, Uq)
                : launch_dependent(hadamard_simt_kernel<kModeY32, false>, grid, dim3(256), 0, st, a, Vq, Uq);
}

}  // namespace wino
