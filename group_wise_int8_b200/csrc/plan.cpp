// Exact construction of the Winograd transforms of F(m,3) from interpolation
// points and diagonal scales ("Data-Free Group-Wise Fully Quantized Winograd
// Convolution via Learnable Scales": B^T = S_B V^{-T}, G = S_G V,
// A^T = V^T S_A with S_A S_B S_G = I; V from homogeneous points, Sec. 7.1).
//
// V_{a x b}[i][j] = f_i^j g_i^(b-1-j) for homogeneous points (f_i, g_i): a
// finite point p is (p, 1), the point at infinity is (1, 0).  V_{nxn} maps the
// coefficients of a degree-(n-1) homogeneous polynomial to its values at the
// points, so column i of V^{-1} holds the coefficients of the Lagrange basis
// polynomial of point i:
//   finite i:  L_i(x) = prod_{k != i, k finite} (x - p_k) / (p_i - p_k)
//   infinity:  L_inf(x) = prod_{k finite} (x - p_k)
// (with the point at infinity present, the finite L_i have degree n-2, so
// they vanish there; L_inf vanishes at every finite point and has leading
// coefficient 1).  Everything is exact rational arithmetic on 128-bit
// integers; each entry is then rounded once to double (one IEEE division of
// exactly representable integers), multiplied by the double scale, and
// rounded to fp32 for B^T and A^T.
#include "plan.h"

#include <cmath>
#include <cstring>

namespace wino {
namespace {

typedef __int128 int128;

struct Q {
    int128 num = 0, den = 1;
};

bool g_bad = false;

int128 abs128(int128 v) { return v < 0 ? -v : v; }

int128 gcd128(int128 a, int128 b) {
    a = abs128(a);
    b = abs128(b);
    while (b) {
        int128 r = a % b;
        a = b;
        b = r;
    }
    return a ? a : 1;
}

Q norm(int128 num, int128 den) {
    if (den == 0) {
        g_bad = true;
        return Q{};
    }
    if (den < 0) {
        num = -num;
        den = -den;
    }
    int128 g = gcd128(num, den);
    Q r;
    r.num = num / g;
    r.den = num == 0 ? 1 : den / g;
    const int128 cap = (int128)1 << 96;
    if (abs128(r.num) > cap || r.den > cap) g_bad = true;
    return r;
}

Q mul(Q a, Q b) {
    int128 g1 = gcd128(a.num, b.den), g2 = gcd128(b.num, a.den);
    return norm((a.num / g1) * (b.num / g2), (a.den / g2) * (b.den / g1));
}

Q add(Q a, Q b) {
    int128 g = gcd128(a.den, b.den);
    return norm(a.num * (b.den / g) + b.num * (a.den / g), a.den / g * b.den);
}

Q neg(Q a) { return Q{-a.num, a.den}; }

Q inv(Q a) { return norm(a.den, a.num); }

// A finite double is m * 2^e with an integer m of at most 53 bits.
bool exact(double x, Q* out) {
    if (!std::isfinite(x)) return false;
    if (x == 0) {
        *out = Q{};
        return true;
    }
    int e;
    double fr = std::frexp(x, &e);
    int128 mant = (int128)(long long)std::ldexp(fr, 53);
    e -= 53;
    if (e > 40 || e < -80) return false;
    *out = e >= 0 ? norm(mant << e, 1) : norm(mant, (int128)1 << (-e));
    return !g_bad;
}

bool to_double(Q q, double* out) {
    const int128 lim = (int128)1 << 53;
    if (abs128(q.num) > lim || q.den > lim) return false;
    *out = (double)(long long)q.num / (double)(long long)q.den;
    return true;
}

// f^j g^(b-1-j) for the homogeneous point
Q vand(bool at_inf, Q p, int j, int b) {
    if (at_inf) return (j == b - 1) ? Q{1, 1} : Q{};
    Q r{1, 1};
    for (int k = 0; k < j; ++k) r = mul(r, p);
    return r;
}

}  // namespace

int build_matrices(int m, const double* points, const float* S_B, const float* S_G, Matrices* out) {
    if ((m != 2 && m != 4 && m != 6) || !points || !out) return WINO_ERR_INVALID_ARG;
    const int n = m + 2;
    g_bad = false;
    bool inf[kMaxN];
    Q p[kMaxN];
    int n_inf = 0;
    for (int i = 0; i < n; ++i) {
        if (std::isnan(points[i])) return WINO_ERR_INVALID_ARG;
        inf[i] = std::isinf(points[i]);
        if (inf[i]) {
            ++n_inf;
            continue;
        }
        if (!exact(points[i], &p[i])) return WINO_ERR_NOT_EXACT;
    }
    if (n_inf > 1) return WINO_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        for (int k = i + 1; k < n; ++k)
            if (!inf[i] && !inf[k] && p[i].num == p[k].num && p[i].den == p[k].den) return WINO_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (S_B && (!std::isfinite(S_B[i]) || S_B[i] == 0.0f)) return WINO_ERR_INVALID_ARG;
        if (S_G && (!std::isfinite(S_G[i]) || S_G[i] == 0.0f)) return WINO_ERR_INVALID_ARG;
    }

    // Vinv[k][i] = coefficient of x^k in L_i
    Q Vinv[kMaxN][kMaxN];
    for (int i = 0; i < n; ++i) {
        Q poly[kMaxN + 1];
        int deg = 0;
        poly[0] = Q{1, 1};
        Q denom{1, 1};
        for (int k = 0; k < n; ++k) {
            if (k == i || inf[k]) continue;
            // poly *= (x - p_k)
            Q next[kMaxN + 1];
            for (int d = 0; d <= deg + 1; ++d) next[d] = Q{};
            for (int d = 0; d <= deg; ++d) {
                next[d + 1] = add(next[d + 1], poly[d]);
                next[d] = add(next[d], mul(neg(p[k]), poly[d]));
            }
            ++deg;
            for (int d = 0; d <= deg; ++d) poly[d] = next[d];
            if (!inf[i]) denom = mul(denom, add(p[i], neg(p[k])));
        }
        if (denom.num == 0) return WINO_ERR_INVALID_ARG;
        Q s = inv(denom);
        for (int k = 0; k < n; ++k) Vinv[k][i] = (k <= deg) ? mul(poly[k], s) : Q{};
    }
    if (g_bad) return WINO_ERR_NOT_EXACT;

    Matrices& M = *out;
    M.m = m;
    M.n = n;
    M.bt_nonzero = M.at_nonzero = 0;
    for (int i = 0; i < n; ++i) {
        double sb = S_B ? (double)S_B[i] : 1.0;
        for (int k = 0; k < n; ++k) {
            double v;
            if (!to_double(Vinv[k][i], &v)) return WINO_ERR_NOT_EXACT;
            M.BT[i * n + k] = (float)(v * sb);
            if (Vinv[k][i].num != 0) M.bt_nonzero |= 1ull << (i * n + k);
        }
    }
    for (int i = 0; i < n; ++i) {
        double sg = S_G ? (double)S_G[i] : 1.0;
        for (int j = 0; j < 3; ++j) {
            double v;
            if (!to_double(vand(inf[i], p[i], j, 3), &v)) return WINO_ERR_NOT_EXACT;
            M.G[i * 3 + j] = v * sg;
        }
    }
    for (int j = 0; j < n; ++j) {
        double sb = S_B ? (double)S_B[j] : 1.0;
        double sg = S_G ? (double)S_G[j] : 1.0;
        double sa = 1.0 / (sb * sg);
        for (int i = 0; i < m; ++i) {
            Q e = vand(inf[j], p[j], i, m);
            double v;
            if (!to_double(e, &v)) return WINO_ERR_NOT_EXACT;
            M.AT[i * n + j] = (float)(v * sa);
            if (e.num != 0) M.at_nonzero |= 1ull << (i * n + j);
        }
    }
    if (g_bad) return WINO_ERR_NOT_EXACT;
    return WINO_OK;
}

namespace {

// One matrix of `len` fp32 entries through the symmetric int8 quantiser, in place.
void quantize_matrix(float* a, int len, uint64_t* nonzero) {
    float amax = 0.0f;
    for (int i = 0; i < len; ++i) amax = std::fmax(amax, std::fabs(a[i]));
    const float s = amax / 127.0f;
    *nonzero = 0;
    for (int i = 0; i < len; ++i) {
        float q = 0.0f;
        if (s != 0.0f) q = std::fmin(127.0f, std::fmax(-127.0f, std::nearbyint(a[i] / s)));
        a[i] = s * q;
        if (a[i] != 0.0f) *nonzero |= 1ull << i;
    }
}

}  // namespace

void quantize_transforms_int8(Matrices* M) {
    quantize_matrix(M->BT, M->n * M->n, &M->bt_nonzero);
    quantize_matrix(M->AT, M->m * M->n, &M->at_nonzero);
}

}  // namespace wino
