// Plain CPU oracle for group-wise fully quantized int8 Winograd convolution F(m,3).
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
// restatement of the method that the CUDA library is checked against.  Only
// the tests, the smoke check and the benchmark's CPU-baseline leg may load it.
// It shares no code, header, table or helper with the CUDA library.
//
// Method source: "Data-Free Group-Wise Fully Quantized Winograd Convolution via
// Learnable Scales" (arXiv 2412.19867), as summarised on its review pages:
//  * transforms from the Vandermonde factorisation B^T = S_B V^{-T},
//    G = S_G V, A^T = V^T S_A with S_A S_B S_G = I ("What carries the
//    argument"; pith extraction "key_machinery");
//  * the homogeneous-point Vandermonde matrix V_{a x b}[i][j] = f_i^j g_i^{b-1-j}
//    (Sec. 7.1 "Standard Winograd transforms");
//  * group-wise int8 quantisation applied to the input transform, the Hadamard
//    product and the output transform (Fig. 2; referee summary (i));
//  * group sizes of 32, 64 or 256 (Sec. 1) and symmetric min-max scaling
//    (assumption "Group-wise quantization with dynamic min-max activation
//    scaling").
//
// Readings taken where the pages are silent (each listed in the design notes):
//  * Q: s = absmax/127 (fp32 IEEE division), q = clamp(rne(v/s), -127, 127),
//    s = 0 and q = 0 for an all-zero group.
//  * V and U groups: G consecutive input channels at a fixed (tile, tap) or
//    (tap, output channel).  Y groups: G consecutive output channels of one
//    tile spanning all n*n taps (the cross-shaped per-tap spread of Y that a
//    single or per-row scale cannot absorb, "Core claim" / Fig. 3).
//  * Fixed fp32 evaluation order (fmaf chains, ascending index, from +0) so that
//    every int8 code is a well-defined function of the inputs.
//  * Alternative readings, selectable (the scales "sqB sqB sqx" of Eqs. (14)-(16),
//    review "Referee Report", minor comment): x through Q per pixel and G
//    consecutive channels (orc_quantize_input); B^T and A^T through Q as one
//    group each (orc_quantize_matrix).  Both leave dequantised fp32 values that
//    the unchanged stages consume.
//
// Parity status: pinned by the CPU tests (exact Winograd identity with
// quantisation off, scale invariance, textbook F(4,3) special case, quantiser
// hand cases, brute-force integer accumulators, grouping properties, hand-written
// codes and scales of the tile-spanning Y requantisation -- ties, a clamp after a
// denormal scale, an all-zero group, maxima at odd taps -- and matmul bounds for
// both output transforms).
//
// Build: g++ -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math).

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- rationals
// Exact rational numbers with 128-bit numerator and denominator.  Points are
// doubles, hence exact dyadic rationals; every Vandermonde entry and every
// entry of its inverse is then an exact rational.
typedef __int128 i128;

struct Rat {
    i128 p, q;  // q > 0, gcd(p, q) = 1
};

bool g_overflow = false;

i128 iabs(i128 a) { return a < 0 ? -a : a; }

i128 igcd(i128 a, i128 b) {
    a = iabs(a);
    b = iabs(b);
    while (b != 0) {
        i128 t = a % b;
        a = b;
        b = t;
    }
    return a;
}

const i128 kLimit = ((i128)1) << 100;

Rat mk(i128 p, i128 q) {
    if (q < 0) {
        p = -p;
        q = -q;
    }
    i128 g = igcd(p, q);
    if (g > 1) {
        p /= g;
        q /= g;
    }
    if (p == 0) q = 1;
    if (iabs(p) > kLimit || q > kLimit) g_overflow = true;
    return Rat{p, q};
}

Rat rmul(Rat a, Rat b) {
    // cross-reduce first to keep the numbers small
    i128 g1 = igcd(a.p, b.q), g2 = igcd(b.p, a.q);
    if (g1 == 0) g1 = 1;
    if (g2 == 0) g2 = 1;
    return mk((a.p / g1) * (b.p / g2), (a.q / g2) * (b.q / g1));
}

Rat rsub(Rat a, Rat b) {
    i128 g = igcd(a.q, b.q);
    i128 l = a.q / g * b.q;
    return mk(a.p * (l / a.q) - b.p * (l / b.q), l);
}

Rat rdiv(Rat a, Rat b) { return rmul(a, mk(b.q, b.p)); }

// exact value of a finite double as a rational
bool rat_from_double(double x, Rat* out) {
    if (!std::isfinite(x)) return false;
    if (x == 0.0) {
        *out = Rat{0, 1};
        return true;
    }
    int e = 0;
    double mant = std::frexp(x, &e);            // x = mant * 2^e, 0.5 <= |mant| < 1
    long long im = (long long)std::ldexp(mant, 53);  // exact: 53-bit integer
    e -= 53;
    // reduce trailing zero bits
    while (im % 2 == 0 && e < 0) {
        im /= 2;
        e += 1;
    }
    if (e > 60 || e < -90) return false;
    i128 p = im, q = 1;
    if (e >= 0)
        p <<= e;
    else
        q <<= -e;
    *out = mk(p, q);
    return !g_overflow;
}

// (double) of a rational: one IEEE division of exactly representable integers
bool rat_to_double(Rat r, double* out) {
    const i128 lim = ((i128)1) << 53;
    if (iabs(r.p) > lim || r.q > lim) return false;
    *out = (double)(long long)r.p / (double)(long long)r.q;
    return true;
}

// ------------------------------------------------------------ plan matrices
// Homogeneous coordinates of a point: a finite point p is (p, 1), the point
// at infinity is (1, 0) (Sec. 7.1).
bool homog(double pt, Rat* f, Rat* g) {
    if (std::isinf(pt)) {
        *f = Rat{1, 1};
        *g = Rat{0, 1};
        return true;
    }
    if (!rat_from_double(pt, f)) return false;
    *g = Rat{1, 1};
    return true;
}

Rat rpow(Rat a, int k) {
    Rat r{1, 1};
    for (int i = 0; i < k; ++i) r = rmul(r, a);
    return r;
}

// V_{a x b}[i][j] = f_i^j * g_i^(b-1-j), i < a, j < b  (Sec. 7.1)
void vandermonde(const std::vector<Rat>& f, const std::vector<Rat>& g, int a, int b,
                 std::vector<Rat>& V) {
    V.assign((size_t)a * b, Rat{0, 1});
    for (int i = 0; i < a; ++i)
        for (int j = 0; j < b; ++j) V[(size_t)i * b + j] = rmul(rpow(f[i], j), rpow(g[i], b - 1 - j));
}

// Gauss-Jordan inverse over the rationals; false if singular.
bool invert(std::vector<Rat> M, int n, std::vector<Rat>& inv) {
    inv.assign((size_t)n * n, Rat{0, 1});
    for (int i = 0; i < n; ++i) inv[(size_t)i * n + i] = Rat{1, 1};
    for (int c = 0; c < n; ++c) {
        int piv = -1;
        for (int r = c; r < n; ++r)
            if (M[(size_t)r * n + c].p != 0) {
                piv = r;
                break;
            }
        if (piv < 0) return false;
        if (piv != c)
            for (int j = 0; j < n; ++j) {
                std::swap(M[(size_t)c * n + j], M[(size_t)piv * n + j]);
                std::swap(inv[(size_t)c * n + j], inv[(size_t)piv * n + j]);
            }
        Rat d = M[(size_t)c * n + c];
        for (int j = 0; j < n; ++j) {
            M[(size_t)c * n + j] = rdiv(M[(size_t)c * n + j], d);
            inv[(size_t)c * n + j] = rdiv(inv[(size_t)c * n + j], d);
        }
        for (int r = 0; r < n; ++r) {
            if (r == c || M[(size_t)r * n + c].p == 0) continue;
            Rat fct = M[(size_t)r * n + c];
            for (int j = 0; j < n; ++j) {
                M[(size_t)r * n + j] = rsub(M[(size_t)r * n + j], rmul(fct, M[(size_t)c * n + j]));
                inv[(size_t)r * n + j] = rsub(inv[(size_t)r * n + j], rmul(fct, inv[(size_t)c * n + j]));
            }
        }
    }
    return true;
}

int g_threads = 0;

void set_omp() {
#ifdef _OPENMP
    if (g_threads > 0) omp_set_num_threads(g_threads);
#endif
}

// ---------------------------------------------------------------- quantiser
// Q over one group (symmetric absmax, int8 range [-127, 127], round half to even).
void quantize_group(const float* v, long stride, int len, signed char* q, long qstride, float* s_out) {
    float amax = 0.0f;
    for (int i = 0; i < len; ++i) {
        float a = std::fabs(v[i * stride]);
        if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    *s_out = s;
    for (int i = 0; i < len; ++i) {
        int qi = 0;
        if (s != 0.0f) {
            float r = std::nearbyint(v[i * stride] / s);  // default rounding mode: half to even
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            qi = (int)r;
        }
        q[i * qstride] = (signed char)qi;
    }
}

}  // namespace

extern "C" {

int orc_set_threads(int t) {
    g_threads = t;
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// Transform matrices of F(m,3) for points[n] (INFINITY = the point at infinity)
// and diagonal scales S_B[n], S_G[n] (NULL = identity).  Outputs (row-major):
//   BT_d, BT_f [n][n]   B^T = S_B V_{nxn}^{-T}
//   G_d        [n][3]   G   = S_G V_{nx3}
//   AT_d, AT_f [m][n]   A^T = V_{nxm}^T S_A,  S_A = (S_B S_G)^{-1}
// Rounding: every exact rational becomes a double by one division; products
// with the scales are double multiplications; the fp32 copies are (float) of
// the doubles.  Returns 0, or -1 (bad m / points), -2 (duplicate points,
// singular V), -3 (rational overflow).
int orc_plan(int m, const double* points, const float* S_B, const float* S_G, double* BT_d,
             float* BT_f, double* G_d, double* AT_d, float* AT_f) {
    if (m < 2 || m > 6 || !points) return -1;
    const int n = m + 2;
    g_overflow = false;
    std::vector<Rat> f(n), g(n);
    for (int i = 0; i < n; ++i)
        if (!homog(points[i], &f[i], &g[i])) return -1;
    std::vector<Rat> Vnn, Vn3, Vnm, Vinv;
    vandermonde(f, g, n, n, Vnn);
    vandermonde(f, g, n, 3, Vn3);
    vandermonde(f, g, n, m, Vnm);
    if (!invert(Vnn, n, Vinv)) return -2;
    if (g_overflow) return -3;
    for (int i = 0; i < n; ++i) {
        double sb = S_B ? (double)S_B[i] : 1.0;
        for (int k = 0; k < n; ++k) {
            double v;
            if (!rat_to_double(Vinv[(size_t)k * n + i], &v)) return -3;  // (V^{-1})^T [i][k]
            double bt = v * sb;
            BT_d[i * n + k] = bt;
            BT_f[i * n + k] = (float)bt;
        }
    }
    for (int i = 0; i < n; ++i) {
        double sg = S_G ? (double)S_G[i] : 1.0;
        for (int j = 0; j < 3; ++j) {
            double v;
            if (!rat_to_double(Vn3[(size_t)i * 3 + j], &v)) return -3;
            G_d[i * 3 + j] = v * sg;
        }
    }
    for (int j = 0; j < n; ++j) {
        double sb = S_B ? (double)S_B[j] : 1.0;
        double sg = S_G ? (double)S_G[j] : 1.0;
        double sa = 1.0 / (sb * sg);
        for (int i = 0; i < m; ++i) {
            double v;
            if (!rat_to_double(Vnm[(size_t)j * m + i], &v)) return -3;
            double at = v * sa;
            AT_d[i * n + j] = at;
            AT_f[i * n + j] = (float)at;
        }
    }
    return 0;
}

// Q on one contiguous group of len values.
void orc_quantize(const float* v, int len, signed char* q, float* s) { quantize_group(v, 1, len, q, 1, s); }

// Alternative reading of the transforms (Eqs. (14)-(16): the input transform
// carries two scales of B): the matrix of len entries as ONE group of Q, each
// entry replaced, in place, by s * q in fp32.
void orc_quantize_matrix(float* a, int len) {
    std::vector<signed char> q(len);
    float s = 0.0f;
    quantize_group(a, 1, len, q.data(), 1, &s);
    for (int i = 0; i < len; ++i) a[i] = s * (float)q[i];
}

// Alternative reading of the input side (same passage: a scale of x): x
// [P][C] (P pixels, NHWC order) through Q per pixel and G consecutive channels,
// each value replaced by s * q in fp32 (xq may alias nothing).
int orc_quantize_input(const float* x, long P, int C, int G, float* xq) {
    if (G <= 0 || C % G != 0) return -1;
    const int ng = C / G;
    set_omp();
#pragma omp parallel
    {
        std::vector<signed char> q(G);
#pragma omp for schedule(static)
        for (long p = 0; p < P; ++p)
            for (int j = 0; j < ng; ++j) {
                const float* v = &x[(size_t)p * C + (size_t)j * G];
                float s = 0.0f;
                quantize_group(v, 1, G, q.data(), 1, &s);
                for (int i = 0; i < G; ++i) xq[(size_t)p * C + (size_t)j * G + i] = s * (float)q[i];
            }
    }
    return 0;
}

// Stage 1: weight transform U = G g G^T per (cout, cin) in fp64 (fma chains,
// ascending index, from +0), U_f = (float)U; then Q over G consecutive input
// channels at fixed (tap, cout).
//   w   [Cout][3][3][Cin] fp32
//   U_f [n*n][Cout][Cin]  fp32 (may be NULL)
//   Uq  [n*n][Cout][Cin]  int8
//   sU  [n*n][Cout][Cin/G] fp32
int orc_weight_transform(int m, const double* G_d, const float* w, int Cin, int Cout, int G,
                         float* U_f, signed char* Uq, float* sU) {
    const int n = m + 2, n2 = n * n;
    if (G <= 0 || Cin % G != 0) return -1;
    const int ng = Cin / G;
    std::vector<float> U((size_t)n2 * Cout * Cin);
    set_omp();
#pragma omp parallel for schedule(static)
    for (int co = 0; co < Cout; ++co) {
        for (int ci = 0; ci < Cin; ++ci) {
            double g[3][3], t[8][3];
            for (int a = 0; a < 3; ++a)
                for (int b = 0; b < 3; ++b) g[a][b] = (double)w[(((size_t)co * 3 + a) * 3 + b) * Cin + ci];
            for (int i = 0; i < n; ++i)
                for (int b = 0; b < 3; ++b) {
                    double acc = 0.0;
                    for (int a = 0; a < 3; ++a) acc = std::fma(G_d[i * 3 + a], g[a][b], acc);
                    t[i][b] = acc;
                }
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    double acc = 0.0;
                    for (int b = 0; b < 3; ++b) acc = std::fma(t[i][b], G_d[j * 3 + b], acc);
                    U[((size_t)(i * n + j) * Cout + co) * Cin + ci] = (float)acc;
                }
        }
    }
    if (U_f) std::memcpy(U_f, U.data(), U.size() * sizeof(float));
    if (!Uq || !sU) return 0;
    for (int tap = 0; tap < n2; ++tap)
        for (int co = 0; co < Cout; ++co)
            for (int j = 0; j < ng; ++j) {
                size_t base = ((size_t)tap * Cout + co) * Cin + (size_t)j * G;
                quantize_group(&U[base], 1, G, &Uq[base], 1, &sU[((size_t)tap * Cout + co) * ng + j]);
            }
    return 0;
}

// Stage 2: input tiles and input transform V = B^T d B in fp32, then Q over G
// consecutive input channels at fixed (tile, tap).
// Tile t = (img*TH + ty)*TW + tx covers input rows ty*m-1 .. ty*m+m and columns
// tx*m-1 .. tx*m+m (zero outside the image: stride 1, pad 1).
//   x   [N][H][W][Cin] fp32 (bf16 inputs are passed widened, exactly)
//   V_f [T][n*n][Cin] fp32 (may be NULL; unquantised transform)
//   Vq  [T][n*n][Cin] int8 (may be NULL)
//   sV  [T][n*n][Cin/G] fp32 (may be NULL)
int orc_input_transform(int m, const float* BT_f, const float* x, int N, int H, int W, int Cin, int G,
                        float* V_f, signed char* Vq, float* sV) {
    const int n = m + 2, n2 = n * n;
    if (G <= 0 || Cin % G != 0) return -1;
    const int TH = (H + m - 1) / m, TW = (W + m - 1) / m;
    const long T = (long)N * TH * TW;
    const int ng = Cin / G;
    set_omp();
#pragma omp parallel
    {
        std::vector<float> Vt((size_t)n2 * Cin);
#pragma omp for schedule(static)
        for (long t = 0; t < T; ++t) {
            const int img = (int)(t / ((long)TH * TW));
            const int ty = (int)((t / TW) % TH), tx = (int)(t % TW);
            for (int c = 0; c < Cin; ++c) {
                float d[8][8], T1[8][8];
                for (int k = 0; k < n; ++k)
                    for (int l = 0; l < n; ++l) {
                        int yy = ty * m - 1 + k, xx = tx * m - 1 + l;
                        d[k][l] = (yy >= 0 && yy < H && xx >= 0 && xx < W)
                                      ? x[(((size_t)img * H + yy) * W + xx) * Cin + c]
                                      : 0.0f;
                    }
                for (int i = 0; i < n; ++i)
                    for (int l = 0; l < n; ++l) {
                        float acc = 0.0f;
                        for (int k = 0; k < n; ++k) acc = std::fmaf(BT_f[i * n + k], d[k][l], acc);
                        T1[i][l] = acc;
                    }
                for (int i = 0; i < n; ++i)
                    for (int j = 0; j < n; ++j) {
                        float acc = 0.0f;
                        for (int l = 0; l < n; ++l) acc = std::fmaf(T1[i][l], BT_f[j * n + l], acc);
                        Vt[(size_t)(i * n + j) * Cin + c] = acc;
                    }
            }
            if (V_f) std::memcpy(&V_f[(size_t)t * n2 * Cin], Vt.data(), Vt.size() * sizeof(float));
            if (Vq && sV)
                for (int tap = 0; tap < n2; ++tap)
                    for (int j = 0; j < ng; ++j)
                        quantize_group(&Vt[(size_t)tap * Cin + (size_t)j * G], 1, G,
                                       &Vq[((size_t)t * n2 + tap) * Cin + (size_t)j * G], 1,
                                       &sV[((size_t)t * n2 + tap) * ng + j]);
        }
    }
    return 0;
}

// Stage 3: Hadamard product summed over input channels, per tap an int8 GEMM
// [T x Cin] . [Cin x Cout].  Per K-group j (G consecutive input channels) the
// exact int32 dot product acc_j is dequantised and accumulated in fp32:
//   y = 0;  for j ascending:  y = fmaf((float)acc_j, sV_j * sU_j, y)
//   Y   [T][n*n][Cout] fp32
//   acc [n*n][T][Cout][Cin/G] int32 (may be NULL)
int orc_hadamard(int n2, const signed char* Vq, const float* sV, const signed char* Uq, const float* sU,
                 long T, int Cin, int Cout, int G, float* Y, int* acc) {
    if (G <= 0 || Cin % G != 0) return -1;
    const int ng = Cin / G;
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t)
        for (int tap = 0; tap < n2; ++tap)
            for (int co = 0; co < Cout; ++co) {
                const signed char* v = &Vq[((size_t)t * n2 + tap) * Cin];
                const signed char* u = &Uq[((size_t)tap * Cout + co) * Cin];
                float y = 0.0f;
                for (int j = 0; j < ng; ++j) {
                    int a = 0;
                    for (int c = j * G; c < (j + 1) * G; ++c) a += (int)v[c] * (int)u[c];
                    if (acc) acc[(((size_t)tap * T + t) * Cout + co) * ng + j] = a;
                    float p = sV[((size_t)t * n2 + tap) * ng + j] * sU[((size_t)tap * Cout + co) * ng + j];
                    y = std::fmaf((float)a, p, y);
                }
                Y[((size_t)t * n2 + tap) * Cout + co] = y;
            }
    return 0;
}

// Stage 4a: requantise Y.  One scale per (tile, block of G consecutive output
// channels) spanning all n*n taps of the tile.
//   Yq [T][n*n][Cout] int8, sY [T][Cout/G] fp32
int orc_y_requant(int n2, const float* Y, long T, int Cout, int G, signed char* Yq, float* sY) {
    if (G <= 0 || Cout % G != 0) return -1;
    const int ng = Cout / G;
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t)
        for (int j = 0; j < ng; ++j) {
            float amax = 0.0f;
            for (int tap = 0; tap < n2; ++tap)
                for (int co = j * G; co < (j + 1) * G; ++co) {
                    float a = std::fabs(Y[((size_t)t * n2 + tap) * Cout + co]);
                    if (a > amax) amax = a;
                }
            float s = amax / 127.0f;
            sY[(size_t)t * ng + j] = s;
            for (int tap = 0; tap < n2; ++tap)
                for (int co = j * G; co < (j + 1) * G; ++co) {
                    int qi = 0;
                    if (s != 0.0f) {
                        float r = std::nearbyint(Y[((size_t)t * n2 + tap) * Cout + co] / s);
                        if (r > 127.0f) r = 127.0f;
                        if (r < -127.0f) r = -127.0f;
                        qi = (int)r;
                    }
                    Yq[((size_t)t * n2 + tap) * Cout + co] = (signed char)qi;
                }
        }
    return 0;
}

// Stage 4a, per-tap reading (Y_TAP): one scale per (tile, tap, block of G
// consecutive couts) instead of one spanning all n*n taps of the tile.
//   Y [T][n2][Cout] fp32 -> Yq [T][n2][Cout] int8, sY [T][n2][Cout/G]
int orc_y_requant_tap(int n2, const float* Y, long T, int Cout, int G, signed char* Yq, float* sY) {
    if (G <= 0 || Cout % G != 0) return -1;
    const int ng = Cout / G;
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t)
        for (int tap = 0; tap < n2; ++tap)
            for (int j = 0; j < ng; ++j) {
                const float* y = Y + ((size_t)t * n2 + tap) * Cout + (size_t)j * G;
                signed char* q = Yq + ((size_t)t * n2 + tap) * Cout + (size_t)j * G;
                quantize_group(y, 1, G, q, 1, &sY[((size_t)t * n2 + tap) * ng + j]);
            }
    return 0;
}

// Stage 4b, per-tap reading: as orc_output_transform, with Yd[xi][nu] scaled by
// the scale of tap (xi, nu).  sY [T][n2][Cout/G]
int orc_output_transform_tap(int m, const float* AT_f, const signed char* Yq, const float* sY, int N, int H,
                             int W, int Cout, int G, float* out) {
    const int n = m + 2, n2 = n * n;
    if (G <= 0 || Cout % G != 0) return -1;
    const int TH = (H + m - 1) / m, TW = (W + m - 1) / m;
    const long T = (long)N * TH * TW;
    const int ng = Cout / G;
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t) {
        const int img = (int)(t / ((long)TH * TW));
        const int ty = (int)((t / TW) % TH), tx = (int)(t % TW);
        for (int co = 0; co < Cout; ++co) {
            float Yd[8][8], Z[8][8];
            for (int xi = 0; xi < n; ++xi)
                for (int nu = 0; nu < n; ++nu) {
                    const int tap = xi * n + nu;
                    const float s = sY[((size_t)t * n2 + tap) * ng + co / G];
                    Yd[xi][nu] = s * (float)Yq[((size_t)t * n2 + tap) * Cout + co];
                }
            for (int i = 0; i < m; ++i)
                for (int nu = 0; nu < n; ++nu) {
                    float acc = 0.0f;
                    for (int xi = 0; xi < n; ++xi) acc = std::fmaf(AT_f[i * n + xi], Yd[xi][nu], acc);
                    Z[i][nu] = acc;
                }
            for (int i = 0; i < m; ++i)
                for (int j = 0; j < m; ++j) {
                    float acc = 0.0f;
                    for (int nu = 0; nu < n; ++nu) acc = std::fmaf(Z[i][nu], AT_f[j * n + nu], acc);
                    int yy = ty * m + i, xx = tx * m + j;
                    if (yy < H && xx < W) out[(((size_t)img * H + yy) * W + xx) * Cout + co] = acc;
                }
        }
    }
    return 0;
}

// Stage 4b: dequantise and output transform, o = A^T (sY * Yq) A, cropped to
// the image.  Z[i][nu] = fmaf-chain over xi of AT[i][xi] * Yd[xi][nu];
// o[i][j] = fmaf-chain over nu of Z[i][nu] * AT[j][nu].
//   out [N][H][W][Cout] fp32
int orc_output_transform(int m, const float* AT_f, const signed char* Yq, const float* sY, int N, int H,
                         int W, int Cout, int G, float* out) {
    const int n = m + 2, n2 = n * n;
    if (G <= 0 || Cout % G != 0) return -1;
    const int TH = (H + m - 1) / m, TW = (W + m - 1) / m;
    const long T = (long)N * TH * TW;
    const int ng = Cout / G;
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t) {
        const int img = (int)(t / ((long)TH * TW));
        const int ty = (int)((t / TW) % TH), tx = (int)(t % TW);
        for (int co = 0; co < Cout; ++co) {
            float s = sY[(size_t)t * ng + co / G];
            float Yd[8][8], Z[8][8];
            for (int xi = 0; xi < n; ++xi)
                for (int nu = 0; nu < n; ++nu)
                    Yd[xi][nu] = s * (float)Yq[((size_t)t * n2 + xi * n + nu) * Cout + co];
            for (int i = 0; i < m; ++i)
                for (int nu = 0; nu < n; ++nu) {
                    float acc = 0.0f;
                    for (int xi = 0; xi < n; ++xi) acc = std::fmaf(AT_f[i * n + xi], Yd[xi][nu], acc);
                    Z[i][nu] = acc;
                }
            for (int i = 0; i < m; ++i)
                for (int j = 0; j < m; ++j) {
                    float acc = 0.0f;
                    for (int nu = 0; nu < n; ++nu) acc = std::fmaf(Z[i][nu], AT_f[j * n + nu], acc);
                    int yy = ty * m + i, xx = tx * m + j;
                    if (yy < H && xx < W) out[(((size_t)img * H + yy) * W + xx) * Cout + co] = acc;
                }
        }
    }
    return 0;
}

// Exact reference: fp64 direct 3x3 correlation, stride 1, pad 1.
//   x [N][H][W][Cin] fp32, w [Cout][3][3][Cin] fp32, out [N][H][W][Cout] fp64
int orc_conv_direct_f64(const float* x, const float* w, int N, int H, int W, int Cin, int Cout, double* out) {
    set_omp();
#pragma omp parallel for collapse(2) schedule(static)
    for (int img = 0; img < N; ++img)
        for (int yy = 0; yy < H; ++yy)
            for (int xx = 0; xx < W; ++xx)
                for (int co = 0; co < Cout; ++co) {
                    double acc = 0.0;
                    for (int a = 0; a < 3; ++a)
                        for (int b = 0; b < 3; ++b) {
                            int iy = yy + a - 1, ix = xx + b - 1;
                            if (iy < 0 || iy >= H || ix < 0 || ix >= W) continue;
                            const float* xp = &x[(((size_t)img * H + iy) * W + ix) * Cin];
                            const float* wp = &w[(((size_t)co * 3 + a) * 3 + b) * Cin];
                            for (int c = 0; c < Cin; ++c) acc += (double)xp[c] * (double)wp[c];
                        }
                    out[(((size_t)img * H + yy) * W + xx) * Cout + co] = acc;
                }
    return 0;
}

// Winograd with quantisation off, in fp64 (BT_d, G_d, AT_d) -- the exact
// transform identity up to fp64 rounding.
int orc_conv_wino_f64(int m, const double* BT_d, const double* G_d, const double* AT_d, const float* x,
                      const float* w, int N, int H, int W, int Cin, int Cout, double* out) {
    const int n = m + 2, n2 = n * n;
    const int TH = (H + m - 1) / m, TW = (W + m - 1) / m;
    const long T = (long)N * TH * TW;
    std::vector<double> U((size_t)n2 * Cout * Cin);
    for (int co = 0; co < Cout; ++co)
        for (int ci = 0; ci < Cin; ++ci) {
            double t[8][3];
            for (int i = 0; i < n; ++i)
                for (int b = 0; b < 3; ++b) {
                    double acc = 0.0;
                    for (int a = 0; a < 3; ++a)
                        acc = std::fma(G_d[i * 3 + a], (double)w[(((size_t)co * 3 + a) * 3 + b) * Cin + ci], acc);
                    t[i][b] = acc;
                }
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    double acc = 0.0;
                    for (int b = 0; b < 3; ++b) acc = std::fma(t[i][b], G_d[j * 3 + b], acc);
                    U[((size_t)(i * n + j) * Cout + co) * Cin + ci] = acc;
                }
        }
    set_omp();
#pragma omp parallel
    {
        std::vector<double> V((size_t)n2 * Cin);
#pragma omp for schedule(static)
        for (long t = 0; t < T; ++t) {
            const int img = (int)(t / ((long)TH * TW));
            const int ty = (int)((t / TW) % TH), tx = (int)(t % TW);
            for (int c = 0; c < Cin; ++c) {
                double d[8][8], T1[8][8];
                for (int k = 0; k < n; ++k)
                    for (int l = 0; l < n; ++l) {
                        int yy = ty * m - 1 + k, xx = tx * m - 1 + l;
                        d[k][l] = (yy >= 0 && yy < H && xx >= 0 && xx < W)
                                      ? (double)x[(((size_t)img * H + yy) * W + xx) * Cin + c]
                                      : 0.0;
                    }
                for (int i = 0; i < n; ++i)
                    for (int l = 0; l < n; ++l) {
                        double acc = 0.0;
                        for (int k = 0; k < n; ++k) acc = std::fma(BT_d[i * n + k], d[k][l], acc);
                        T1[i][l] = acc;
                    }
                for (int i = 0; i < n; ++i)
                    for (int j = 0; j < n; ++j) {
                        double acc = 0.0;
                        for (int l = 0; l < n; ++l) acc = std::fma(T1[i][l], BT_d[j * n + l], acc);
                        V[(size_t)(i * n + j) * Cin + c] = acc;
                    }
            }
            for (int co = 0; co < Cout; ++co) {
                double Y[8][8], Z[8][8];
                for (int tap = 0; tap < n2; ++tap) {
                    double acc = 0.0;
                    for (int c = 0; c < Cin; ++c)
                        acc = std::fma(V[(size_t)tap * Cin + c], U[((size_t)tap * Cout + co) * Cin + c], acc);
                    Y[tap / n][tap % n] = acc;
                }
                for (int i = 0; i < m; ++i)
                    for (int nu = 0; nu < n; ++nu) {
                        double acc = 0.0;
                        for (int xi = 0; xi < n; ++xi) acc = std::fma(AT_d[i * n + xi], Y[xi][nu], acc);
                        Z[i][nu] = acc;
                    }
                for (int i = 0; i < m; ++i)
                    for (int j = 0; j < m; ++j) {
                        double acc = 0.0;
                        for (int nu = 0; nu < n; ++nu) acc = std::fma(Z[i][nu], AT_d[j * n + nu], acc);
                        int yy = ty * m + i, xx = tx * m + j;
                        if (yy < H && xx < W) out[(((size_t)img * H + yy) * W + xx) * Cout + co] = acc;
                    }
            }
        }
    }
    return 0;
}

// Winograd with quantisation off, in fp32 with the same evaluation order as
// the quantised pipeline (Y accumulated channel by channel with fmaf).
int orc_conv_wino_f32(int m, const float* BT_f, const double* G_d, const float* AT_f, const float* x,
                      const float* w, int N, int H, int W, int Cin, int Cout, float* out) {
    const int n = m + 2, n2 = n * n;
    const int TH = (H + m - 1) / m, TW = (W + m - 1) / m;
    const long T = (long)N * TH * TW;
    std::vector<float> U((size_t)n2 * Cout * Cin), V((size_t)T * n2 * Cin);
    orc_weight_transform(m, G_d, w, Cin, Cout, Cin, U.data(), nullptr, nullptr);
    orc_input_transform(m, BT_f, x, N, H, W, Cin, Cin, V.data(), nullptr, nullptr);
    set_omp();
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; ++t) {
        const int img = (int)(t / ((long)TH * TW));
        const int ty = (int)((t / TW) % TH), tx = (int)(t % TW);
        for (int co = 0; co < Cout; ++co) {
            float Y[8][8], Z[8][8];
            for (int tap = 0; tap < n2; ++tap) {
                float acc = 0.0f;
                for (int c = 0; c < Cin; ++c)
                    acc = std::fmaf(V[((size_t)t * n2 + tap) * Cin + c], U[((size_t)tap * Cout + co) * Cin + c], acc);
                Y[tap / n][tap % n] = acc;
            }
            for (int i = 0; i < m; ++i)
                for (int nu = 0; nu < n; ++nu) {
                    float acc = 0.0f;
                    for (int xi = 0; xi < n; ++xi) acc = std::fmaf(AT_f[i * n + xi], Y[xi][nu], acc);
                    Z[i][nu] = acc;
                }
            for (int i = 0; i < m; ++i)
                for (int j = 0; j < m; ++j) {
                    float acc = 0.0f;
                    for (int nu = 0; nu < n; ++nu) acc = std::fmaf(Z[i][nu], AT_f[j * n + nu], acc);
                    int yy = ty * m + i, xx = tx * m + j;
                    if (yy < H && xx < W) out[(((size_t)img * H + yy) * W + xx) * Cout + co] = acc;
                }
        }
    }
    return 0;
}

}  // extern "C"
