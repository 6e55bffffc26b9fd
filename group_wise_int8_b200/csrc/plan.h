// Host-side transform plan of the Winograd library (internal header).
#pragma once
#include <cstdint>

#include "../../include/wino.h"

namespace wino {

constexpr int kMaxN = 8;  // n = m + 2 <= 8

struct Matrices {
    int m = 0, n = 0;
    float BT[kMaxN * kMaxN];   // B^T  [n][n]
    double G[kMaxN * 3];       // G    [n][3]
    float AT[6 * kMaxN];       // A^T  [m][n]
    uint64_t bt_nonzero = 0;   // bit i*n+k set iff B^T[i][k] != 0 (exact)
    uint64_t at_nonzero = 0;   // bit i*n+j set iff A^T[i][j] != 0 (exact)
};

// Builds B^T = S_B V^{-T}, G = S_G V_{nx3}, A^T = V_{nxm}^T S_A for F(m,3).
// Returns WINO_OK, WINO_ERR_INVALID_ARG or WINO_ERR_NOT_EXACT.
int build_matrices(int m, const double* points, const float* S_B, const float* S_G, Matrices* out);

// Int8 transforms with one scale per matrix: B^T and A^T each become s * q, where
// s = max|entry| / 127 (fp32 division), q = clamp(rne(entry / s), +-127), the product
// rounded to fp32.  The nonzero masks are recomputed from the quantised entries.
void quantize_transforms_int8(Matrices* M);

}  // namespace wino
