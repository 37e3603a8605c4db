// TurboQuant-style KV-cache compressor: plain scalar fp64 CPU ORACLE.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
// this file.  It exists so that tests, the smoke check and the CPU-baseline leg
// of the benchmark can check the CUDA library against an independent, slow,
// obviously-correct restatement of the method.  It shares no code, header,
// table or constant generator with the CUDA library.
//
// Sources (cited by page title and section):
//   [FQ-TQ]  "FlashQuant：生产级KV缓存压缩方案，让大模型推理显存占用降低7.5倍"
//            (zingnex.cn forum thread flashquant-kv-7-5)
//            - section "TurboQuant：Google Research的突破性算法": the four steps
//              normalize / rotate by R^T / Lloyd-Max (Gaussian) / pack nibbles +
//              fp32 norm, and the MSE bound (sqrt(3)*pi/2)/4^b * ||x||^2.
//            - section "注意力计算的特殊挑战与QJL校正": the QJL estimator
//              <q,k> ~ <q,k_mse> + gamma*sqrt(pi/2)/d*<Sq, sign(Sr)>, r = k - k_mse,
//              gamma = ||r||, S a random sign matrix, one extra bit per dimension.
//            - section "架构设计": Codebook (Lloyd-Max), Quantizer (MSE / Prod modes),
//              Packing (nibble / 2-bit), Rotation (Haar QR).
//   [TQ-RS]  "TurboQuant : compresser le KV-cache des LLM par 7x sans perdre en
//            qualité" (patricehuetz.fr)
//            - "Couche 1": randomized Walsh-Hadamard rotation (signs, butterflies,
//              scale 1/sqrt(n)).
//            - "Couche 3": 2 indices per byte at 4 bits, 4 per byte at 2 bits.
//            - "Couche 4": the norm kept separately in fp32 (4 bytes per vector).
//
// Readings of points the pages leave open are marked READING below; every one of
// them is listed in the repository's design notes.
//
// Parity status: every function here is pinned by the CPU test-suite against
// closed forms, invariants, library routines or brute force (no function is
// "parity unpinned").

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------------------
// Random numbers.  READING: the pages fix no generator.  Every seeded draw of
// the method (Haar Gaussian matrix, QJL signs, Hadamard signs) comes from a
// SplitMix64 stream (Steele, Lea & Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014).  Stream (seed, tag) starts from state
// seed + tag * 2^48; tag 0 = Haar Gaussian matrix, 1 = QJL matrix S,
// 2 = Hadamard signs.
// ---------------------------------------------------------------------------
struct Stream {
    uint64_t state;
    Stream(uint64_t seed, uint64_t tag) : state(seed + (tag << 48)) {}
    uint64_t next() {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
    // uniform on the open interval (0, 1): the top 53 bits, centred in their cell
    double uniform() { return ((double)(next() >> 11) + 0.5) * (1.0 / 9007199254740992.0); }
    // +1 when the top bit of the word is 0, -1 otherwise
    int sign() { return (next() >> 63) ? -1 : 1; }
};

// Box-Muller: two uniforms give two independent standard normals, used in order.
void gaussian_fill(uint64_t seed, uint64_t tag, long count, double* out) {
    Stream s(seed, tag);
    const double two_pi = 6.283185307179586476925286766559;
    for (long k = 0; k < count; k += 2) {
        double u1 = s.uniform();
        double u2 = s.uniform();
        double rad = std::sqrt(-2.0 * std::log(u1));
        out[k] = rad * std::cos(two_pi * u2);
        if (k + 1 < count) out[k + 1] = rad * std::sin(two_pi * u2);
    }
}

void sign_fill(uint64_t seed, uint64_t tag, long count, int8_t* out) {
    Stream s(seed, tag);
    for (long k = 0; k < count; ++k) out[k] = (int8_t)s.sign();
}

// ---------------------------------------------------------------------------
// Haar rotation [FQ-TQ "架构设计": Rotation (Haar QR矩阵)].
// G ~ N(0,1)^{d x d} (row-major from stream tag 0); G = QR by Householder
// reflections; READING: plain QR is Haar-distributed only once the columns of Q
// are multiplied by sign(diag(R)), so that R has a positive diagonal; that is
// the matrix used.  Convention [FQ-TQ step 2 applies R^T]: y = R^T x.
// Output Rm is row-major: Rm[i*d + j] = R_{ij}.
// ---------------------------------------------------------------------------
void haar_rotation(int d, uint64_t seed, double* Rm) {
    std::vector<double> A((size_t)d * d);
    gaussian_fill(seed, 0, (long)d * d, A.data());
    std::vector<double> V((size_t)d * d, 0.0);   // Householder vectors, column k in V[:,k]
    std::vector<double> alpha(d);
    for (int k = 0; k < d; ++k) {
        double nrm2 = 0.0;
        for (int i = k; i < d; ++i) nrm2 += A[(size_t)i * d + k] * A[(size_t)i * d + k];
        double nrm = std::sqrt(nrm2);
        double x0 = A[(size_t)k * d + k];
        double a = (x0 >= 0.0) ? -nrm : nrm;      // R_kk of this QR
        alpha[k] = a;
        // v = x - a e_1, normalised
        std::vector<double> v(d, 0.0);
        for (int i = k; i < d; ++i) v[i] = A[(size_t)i * d + k];
        v[k] -= a;
        double vn2 = 0.0;
        for (int i = k; i < d; ++i) vn2 += v[i] * v[i];
        double vn = std::sqrt(vn2);
        if (vn > 0.0)
            for (int i = k; i < d; ++i) v[i] /= vn;
        for (int i = 0; i < d; ++i) V[(size_t)i * d + k] = v[i];
        // A[k:, k:] -= 2 v (v^T A[k:, k:])
        for (int j = k; j < d; ++j) {
            double dot = 0.0;
            for (int i = k; i < d; ++i) dot += v[i] * A[(size_t)i * d + j];
            for (int i = k; i < d; ++i) A[(size_t)i * d + j] -= 2.0 * v[i] * dot;
        }
    }
    // Q = H_0 H_1 ... H_{d-1}; build it by applying the reflections to I from the right end.
    std::vector<double> Q((size_t)d * d, 0.0);
    for (int i = 0; i < d; ++i) Q[(size_t)i * d + i] = 1.0;
    for (int k = d - 1; k >= 0; --k) {
        for (int j = 0; j < d; ++j) {
            double dot = 0.0;
            for (int i = k; i < d; ++i) dot += V[(size_t)i * d + k] * Q[(size_t)i * d + j];
            for (int i = k; i < d; ++i) Q[(size_t)i * d + j] -= 2.0 * V[(size_t)i * d + k] * dot;
        }
    }
    // sign fix: column k times sign(R_kk)
    for (int k = 0; k < d; ++k) {
        double s = (alpha[k] < 0.0) ? -1.0 : 1.0;
        for (int i = 0; i < d; ++i) Rm[(size_t)i * d + k] = Q[(size_t)i * d + k] * s;
    }
}

// ---------------------------------------------------------------------------
// Randomized Walsh-Hadamard rotation [TQ-RS "Couche 1"]: multiply by the +-1
// signs, run the in-place butterflies with strides 1, 2, 4, ..., divide by
// sqrt(n).  In matrix form y = H D x / sqrt(d) with H the Sylvester-ordered
// Hadamard matrix, so R^T = H D / sqrt(d) and R = D H / sqrt(d).
// ---------------------------------------------------------------------------
void fwht_inplace(int n, double* x) {
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = x[j], b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
}

void hadamard_rotation_matrix(int d, const int8_t* D, double* Rm) {
    // column j of R^T H D / sqrt(d) applied to e_i gives row i of R^T; build R directly:
    // R^T e_i = H D e_i / sqrt(d)  ->  column i of R^T = row i of R.
    std::vector<double> e(d);
    for (int i = 0; i < d; ++i) {
        for (int k = 0; k < d; ++k) e[k] = 0.0;
        e[i] = (double)D[i];
        fwht_inplace(d, e.data());
        for (int j = 0; j < d; ++j) Rm[(size_t)i * d + j] = e[j] / std::sqrt((double)d);
    }
}

// ---------------------------------------------------------------------------
// Gaussian Lloyd-Max scalar quantizer [FQ-TQ step 3: "高斯分布有闭式解"].
// READING: only the 1-bit case has a closed form; for b >= 2 the codebook is
// the fixed point of Lloyd's two conditions, each of which is evaluated in
// closed form for the unit normal law:
//   centroid  c_j = (phi(t_j) - phi(t_{j+1})) / (Phi(t_{j+1}) - Phi(t_j))
//   boundary  t_j = (c_{j-1} + c_j) / 2
// with t_0 = -inf, t_L = +inf.  Iterated in fp64 until nothing moves by more
// than 1e-15 (or 200000 rounds).  c has L = 2^b entries, t has L-1 interior
// boundaries.
// ---------------------------------------------------------------------------
double npdf(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * 3.14159265358979323846); }
// P(a < X < b) for X ~ N(0,1), using the tail form on whichever side keeps precision
double cell_prob(double a, double b) {
    const double r2 = 1.4142135623730950488016887242097;
    if (a >= 0.0) return 0.5 * (std::erfc(a / r2) - std::erfc(b / r2));
    if (b <= 0.0) return 0.5 * (std::erfc(-b / r2) - std::erfc(-a / r2));
    return 1.0 - 0.5 * std::erfc(-a / r2) - 0.5 * std::erfc(b / r2);   // 1 - Phi(a) - Q(b)
}

void lloyd_max_gaussian(int bits, double* c, double* t) {
    const int L = 1 << bits;
    std::vector<double> cc(L), tt(L + 1);
    // start from evenly spaced centroids on [-2, 2]
    for (int j = 0; j < L; ++j) cc[j] = (L == 1) ? 0.0 : -2.0 + 4.0 * (j + 0.5) / L;
    const double inf = INFINITY;
    for (int it = 0; it < 200000; ++it) {
        tt[0] = -inf;
        tt[L] = inf;
        for (int j = 1; j < L; ++j) tt[j] = 0.5 * (cc[j - 1] + cc[j]);
        double moved = 0.0;
        for (int j = 0; j < L; ++j) {
            double a = tt[j], b = tt[j + 1];
            double pa = std::isinf(a) ? 0.0 : npdf(a);
            double pb = std::isinf(b) ? 0.0 : npdf(b);
            double nc = (pa - pb) / cell_prob(a, b);
            double dm = std::fabs(nc - cc[j]);
            if (dm > moved) moved = dm;
            cc[j] = nc;
        }
        if (moved < 1e-15) break;
    }
    for (int j = 0; j < L; ++j) c[j] = cc[j];
    for (int j = 1; j < L; ++j) t[j - 1] = 0.5 * (cc[j - 1] + cc[j]);
}

// ---------------------------------------------------------------------------
// Exact-d codebook ([TQ-RS] "Étape 2" and "Couche 2": after the rotation each
// coordinate of a unit vector follows the spherical Beta law, and the Lloyd-Max
// quantizer is computed for that law).  The coordinate compared with the
// boundaries is v = sqrt(d) u_1, u uniform on the unit sphere of R^d, whose
// density is proportional to (1 - v^2/d)^((d-3)/2) on (-sqrt(d), sqrt(d)).
// Lloyd's two conditions, as for the Gaussian codebook:
//   c_j = int_{t_j}^{t_{j+1}} v f(v) dv / int_{t_j}^{t_{j+1}} f(v) dv,
//   t_j = (c_{j-1} + c_j) / 2,
// the numerator in closed form, -d/(d-1) (1 - v^2/d)^((d-1)/2) / Z between the
// cell's ends, the denominator through the law's CDF, a regularized incomplete
// beta function: (u_1 + 1) / 2 ~ Beta((d-1)/2, (d-1)/2).  READING: the page's "50 iterations" do not converge in
// fp64; iterated, like the Gaussian codebook, until nothing moves by 1e-15.
// ---------------------------------------------------------------------------
// Regularized incomplete beta I_x(p, q) by its continued fraction (DLMF 8.17.22,
// evaluated with the modified Lentz method), for x < (p + 1) / (p + q + 2).
double ibeta_cf(double x, double p, double q) {
    const double lead = std::exp(p * std::log(x) + q * std::log1p(-x) -
                                 (std::lgamma(p) + std::lgamma(q) - std::lgamma(p + q))) / p;
    const double tiny = 1e-300;
    double f = 1.0, C = 1.0, Dn = 0.0;
    for (int i = 0; i <= 4000; ++i) {
        double num;
        if (i == 0) {
            num = 1.0;
        } else {
            const int m = i / 2;
            num = (i & 1) ? -((p + m) * (p + q + m) * x) / ((p + 2.0 * m) * (p + 2.0 * m + 1.0))
                          : (m * (q - m) * x) / ((p + 2.0 * m - 1.0) * (p + 2.0 * m));
        }
        Dn = 1.0 + num * Dn;
        if (std::fabs(Dn) < tiny) Dn = tiny;
        Dn = 1.0 / Dn;
        C = 1.0 + num / C;
        if (std::fabs(C) < tiny) C = tiny;
        const double delta = C * Dn;
        f *= delta;
        if (std::fabs(delta - 1.0) < 1e-16) break;
    }
    return lead * (f - 1.0);
}
// P(V > v) for v >= 0: V = sqrt(d) u_1, (u_1 + 1) / 2 ~ Beta((d-1)/2, (d-1)/2)
double beta_upper_tail(int d, double v) {
    const double p = 0.5 * (d - 1);
    const double x = 0.5 * (1.0 - v / std::sqrt((double)d));   // P(V > v) = I_x(p, p)
    if (x <= 0.0) return 0.0;
    return ibeta_cf(x, p, p);   // x <= 1/2 < (p + 1) / (2p + 2)
}
// int_a^b of the density (normalised), on the side of 0 that keeps precision
double beta_mass(int d, double a, double b) {
    if (a >= 0.0) return beta_upper_tail(d, a) - beta_upper_tail(d, b);
    if (b <= 0.0) return beta_upper_tail(d, -b) - beta_upper_tail(d, -a);
    return 1.0 - beta_upper_tail(d, -a) - beta_upper_tail(d, b);
}
// int_a^b v f(v) dv for the normalised density f(v) = (1 - v^2/d)^((d-3)/2) / Z,
// Z = sqrt(d) B(1/2, (d-1)/2); the antiderivative is -d/(d-1) (1 - v^2/d)^((d-1)/2) / Z
double beta_first_moment(int d, double a, double b) {
    const double k1 = 0.5 * (d - 1);
    const double logZ = 0.5 * std::log((double)d) + std::lgamma(0.5) + std::lgamma(k1) - std::lgamma(0.5 + k1);
    auto F = [&](double v) {
        const double w = 1.0 - v * v / d;
        return w <= 0.0 ? 0.0 : -(double)d / (d - 1) * std::exp(k1 * std::log(w) - logZ);
    };
    return F(b) - F(a);
}

void lloyd_max_beta(int d, int bits, double* c, double* t) {
    const int L = 1 << bits;
    const double vmax = std::sqrt((double)d);
    std::vector<double> cc(L), tt(L + 1);
    for (int j = 0; j < L; ++j) cc[j] = (L == 1) ? 0.0 : -2.0 + 4.0 * (j + 0.5) / L;
    for (int it = 0; it < 200000; ++it) {
        tt[0] = -vmax;
        tt[L] = vmax;
        for (int j = 1; j < L; ++j) tt[j] = 0.5 * (cc[j - 1] + cc[j]);
        double moved = 0.0;
        for (int j = 0; j < L; ++j) {
            const double nc = beta_first_moment(d, tt[j], tt[j + 1]) / beta_mass(d, tt[j], tt[j + 1]);
            const double dm = std::fabs(nc - cc[j]);
            if (dm > moved) moved = dm;
            cc[j] = nc;
        }
        if (moved < 1e-15) break;
    }
    for (int j = 0; j < L; ++j) c[j] = cc[j];
    for (int j = 1; j < L; ++j) t[j - 1] = 0.5 * (cc[j - 1] + cc[j]);
}

// ---------------------------------------------------------------------------
// Packed layout of one 16-token page chunk (READING: the pages fix only the
// nibble / 2-bit packing and the separate fp32 norm; byte and bit order, the
// 1-bit container and the per-chunk arrangement are this design's):
//   container width w(b) = 4 for b in {3,4}, 2 for b = 2, 1 for b = 1
//   MSE chunk:  codes[16][d*w/8] | norm f32[16]
//   prod chunk: codes[16][d*w/8] | signs[16][d/8] | norm f32[16] | gamma f32[16]
//   nibble: byte i = c[2i] | c[2i+1] << 4; crumb: byte i = sum_k c[4i+k] << 2k;
//   bit:    byte i = sum_k c[8i+k] << k
// ---------------------------------------------------------------------------
// Dense 3-bit option ([TQ-RS] "Couche 3" packs indices into bytes; the dense form
// is this design's): 3-bit codes as a bit string, code i in bits [3i, 3i + 3),
// least significant bit first -- 48 B per 128 codes instead of 64 B of nibbles.
int container_width(int b) { return b >= 3 ? 4 : (b == 2 ? 2 : 1); }
int code_width(int b, bool dense3) { return (dense3 && b == 3) ? 3 : container_width(b); }

// codes as a bit string: code i occupies bits [w i, w i + w) of out, LSB first
// (for w = 1, 2, 4 this is byte i = sum_k c[(8/w) i + k] << k w)
void pack_codes(const int* codes, int n, int w, uint8_t* out) {
    const int nbytes = n * w / 8;
    for (int i = 0; i < nbytes; ++i) out[i] = 0;
    for (int i = 0; i < n; ++i)
        for (int k = 0; k < w; ++k)
            if ((codes[i] >> k) & 1) out[(i * w + k) / 8] |= (uint8_t)(1u << ((i * w + k) % 8));
}

void unpack_codes(const uint8_t* in, int n, int w, int* codes) {
    for (int i = 0; i < n; ++i) {
        int c = 0;
        for (int k = 0; k < w; ++k) c |= ((in[(i * w + k) / 8] >> ((i * w + k) % 8)) & 1) << k;
        codes[i] = c;
    }
}

struct Params {
    int d, bits, rot, key_mode;   // rot: 0 Haar, 1 Hadamard; key_mode: 0 prod (QJL), 1 MSE
    int beta = 0;                 // codebooks: 0 Gaussian Lloyd-Max, 1 exact-d (spherical Beta) Lloyd-Max
    int dense3 = 0;               // 3-bit codes: 0 nibble containers, 1 dense bit string
    std::vector<double> R;        // row-major, y = R^T x
    std::vector<int8_t> S;        // row-major, (S r)_j = sum_i S[j][i] r_i
    std::vector<int8_t> D;        // Hadamard signs (rot == 1)
    int vbits, kbits;             // code bits of values and keys
    std::vector<double> cv, tv;   // value codebook / boundaries
    std::vector<double> ck, tk;   // key codebook / boundaries
};

size_t chunk_bytes(const Params& P, int kind /*0 key, 1 value*/) {
    const int d = P.d;
    if (kind == 1 || P.key_mode == 1) {
        int b = (kind == 1) ? P.vbits : P.kbits;
        return (size_t)16 * d * code_width(b, P.dense3) / 8 + 64;
    }
    return (size_t)16 * d * code_width(P.kbits, P.dense3) / 8 + (size_t)16 * d / 8 + 128;
}

// One vector through the compress step [FQ-TQ steps 1-4, QJL section].
// Outputs: codes[d], norm, and for prod keys signs[d] (0/1) and gamma.
// Diagnostics (may be null): v[d] = sqrt(d)*u_i (the value compared to the
// boundaries) and sk[d] = (S r)_j / n.
struct VecOut {
    double norm = 0, gamma = 0;
};

VecOut compress_vector(const Params& P, int kind, const double* x, int* codes, int* signs,
                       double* v_diag, double* sk_diag) {
    const int d = P.d;
    const bool value = (kind == 1);
    const bool prod = !value && P.key_mode == 0;
    const int b = value ? P.vbits : P.kbits;
    const int L = 1 << b;
    const std::vector<double>& c = value ? P.cv : P.ck;
    const std::vector<double>& t = value ? P.tv : P.tk;
    VecOut o;
    // step 1: norm and direction
    double n2 = 0.0;
    for (int i = 0; i < d; ++i) n2 += x[i] * x[i];
    const double n = std::sqrt(n2);
    o.norm = n;
    if (n == 0.0) {
        // READING: a zero vector takes the cell of 0 (t = 0 is a boundary and is
        // not counted), all signs 1 (sign(0) = +1), gamma 0.
        for (int i = 0; i < d; ++i) {
            codes[i] = L / 2 - 1;
            if (v_diag) v_diag[i] = 0.0;
        }
        if (prod)
            for (int j = 0; j < d; ++j) {
                signs[j] = 1;
                if (sk_diag) sk_diag[j] = 0.0;
            }
        o.gamma = 0.0;
        return o;
    }
    // step 2: rotate, y = R^T x; u = y / n
    std::vector<double> u(d);
    for (int j = 0; j < d; ++j) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += P.R[(size_t)i * d + j] * x[i];
        u[j] = s / n;
    }
    // step 3: Lloyd-Max on the unit-variance coordinate sqrt(d)*u_j;
    // idx = #{ interior boundaries strictly below the value } (READING: ties go low)
    const double sd = std::sqrt((double)d);
    for (int j = 0; j < d; ++j) {
        double v = sd * u[j];
        int idx = 0;
        for (int k = 0; k < L - 1; ++k)
            if (t[k] < v) ++idx;
        codes[j] = idx;
        if (v_diag) v_diag[j] = v;
    }
    if (!prod) return o;
    // QJL [FQ-TQ QJL section]: k_mse = n * R * (c[idx] / sqrt(d)); r = x - k_mse;
    // gamma = ||r||; sign bit j = 1 iff (S r)_j >= 0.
    std::vector<double> khat(d), r(d);
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += P.R[(size_t)i * d + j] * c[codes[j]];
        khat[i] = n * s / sd;
    }
    double g2 = 0.0;
    for (int i = 0; i < d; ++i) {
        r[i] = x[i] - khat[i];
        g2 += r[i] * r[i];
    }
    o.gamma = std::sqrt(g2);
    for (int j = 0; j < d; ++j) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += (double)P.S[(size_t)j * d + i] * r[i];
        signs[j] = (s >= 0.0) ? 1 : 0;
        if (sk_diag) sk_diag[j] = s / n;
    }
    return o;
}

// Decompress one vector from its unpacked fields.
// MSE: x_hat = n * R * c[idx] / sqrt(d).
// READING (keys, prod): the vector whose inner product with any q equals the
// QJL estimator, k_tilde = k_hat + gamma*sqrt(pi/2)/d * S^T (2 sigma - 1).
void decompress_vector(const Params& P, int kind, const int* codes, const int* signs, double norm,
                       double gamma, double* out) {
    const int d = P.d;
    const bool value = (kind == 1);
    const bool prod = !value && P.key_mode == 0;
    const std::vector<double>& c = value ? P.cv : P.ck;
    const double sd = std::sqrt((double)d);
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += P.R[(size_t)i * d + j] * c[codes[j]];
        out[i] = norm * s / sd;
    }
    if (!prod) return;
    const double coef = gamma * std::sqrt(3.14159265358979323846 / 2.0) / d;
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += (double)P.S[(size_t)j * d + i] * (2.0 * signs[j] - 1.0);
        out[i] += coef * s;
    }
}

// Read the fields of one (chunk, row) from a packed cache.
void read_row(const Params& P, int kind, const uint8_t* chunk, int row, int* codes, int* signs,
              double* norm, double* gamma) {
    const int d = P.d;
    const bool value = (kind == 1);
    const bool prod = !value && P.key_mode == 0;
    const int b = value ? P.vbits : P.kbits;
    const int w = code_width(b, P.dense3);
    const size_t code_row = (size_t)d * w / 8;
    unpack_codes(chunk + row * code_row, d, w, codes);
    size_t off = 16 * code_row;
    if (prod) {
        unpack_codes(chunk + off + (size_t)row * (d / 8), d, 1, signs);
        off += (size_t)16 * (d / 8);
    }
    float nf, gf = 0.f;
    std::memcpy(&nf, chunk + off + 4 * row, 4);
    if (prod) std::memcpy(&gf, chunk + off + 64 + 4 * row, 4);
    *norm = nf;
    *gamma = gf;
}

void write_row(const Params& P, int kind, uint8_t* chunk, int row, const int* codes, const int* signs,
               double norm, double gamma) {
    const int d = P.d;
    const bool value = (kind == 1);
    const bool prod = !value && P.key_mode == 0;
    const int b = value ? P.vbits : P.kbits;
    const int w = code_width(b, P.dense3);
    const size_t code_row = (size_t)d * w / 8;
    pack_codes(codes, d, w, chunk + row * code_row);
    size_t off = 16 * code_row;
    if (prod) {
        pack_codes(signs, d, 1, chunk + off + (size_t)row * (d / 8));
        off += (size_t)16 * (d / 8);
    }
    float nf = (float)norm;   // stored fp32 [FQ-TQ step 4; TQ-RS Couche 4]
    std::memcpy(chunk + off + 4 * row, &nf, 4);
    if (prod) {
        float gf = (float)gamma;
        std::memcpy(chunk + off + 64 + 4 * row, &gf, 4);
    }
}

void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

}  // namespace

extern "C" {

// ---- primitives exposed for the pins -------------------------------------
void orc_splitmix64(uint64_t seed, uint64_t tag, long count, uint64_t* out) {
    Stream s(seed, tag);
    for (long k = 0; k < count; ++k) out[k] = s.next();
}
void orc_uniform(uint64_t seed, uint64_t tag, long count, double* out) {
    Stream s(seed, tag);
    for (long k = 0; k < count; ++k) out[k] = s.uniform();
}
void orc_gaussian(uint64_t seed, uint64_t tag, long count, double* out) { gaussian_fill(seed, tag, count, out); }
void orc_signs(uint64_t seed, uint64_t tag, long count, int8_t* out) { sign_fill(seed, tag, count, out); }
void orc_haar(int d, uint64_t seed, double* R) { haar_rotation(d, seed, R); }
void orc_fwht(int n, double* x) { fwht_inplace(n, x); }
void orc_hadamard_matrix(int d, const int8_t* D, double* R) { hadamard_rotation_matrix(d, D, R); }
void orc_lloyd_max(int bits, double* c, double* t) { lloyd_max_gaussian(bits, c, t); }
void orc_pack(const int* codes, int n, int w, uint8_t* out) { pack_codes(codes, n, w, out); }
void orc_unpack(const uint8_t* in, int n, int w, int* codes) { unpack_codes(in, n, w, codes); }

// ---- parameters ------------------------------------------------------------
// rot: 0 = Haar, 1 = randomized Hadamard.  key_mode: 0 = prod (b-1 bit MSE code
// + 1-bit QJL), 1 = MSE at b bits.  d must be a power of two >= 8.
void orc_lloyd_max_beta(int d, int bits, double* c, double* t) { lloyd_max_beta(d, bits, c, t); }

void* orc_create_ex(int d, int bits, uint64_t seed, int rot, int key_mode, int beta, int dense3);
void* orc_create(int d, int bits, uint64_t seed, int rot, int key_mode) {
    return orc_create_ex(d, bits, seed, rot, key_mode, 0, 0);
}

// beta: exact-d codebooks instead of the Gaussian ones; dense3: 3-bit codes as a
// dense bit string instead of nibbles (both READINGS of [TQ-RS] "Couche 2" / "Couche 3").
void* orc_create_ex(int d, int bits, uint64_t seed, int rot, int key_mode, int beta, int dense3) {
    if (d < 8 || (d & (d - 1)) != 0 || bits < 1 || bits > 8) return nullptr;
    if (key_mode == 0 && bits < 2) return nullptr;
    Params* P = new Params();
    P->d = d;
    P->bits = bits;
    P->rot = rot;
    P->key_mode = key_mode;
    P->R.resize((size_t)d * d);
    if (rot == 0) {
        haar_rotation(d, seed, P->R.data());
    } else {
        P->D.resize(d);
        sign_fill(seed, 2, d, P->D.data());
        hadamard_rotation_matrix(d, P->D.data(), P->R.data());
    }
    // READING: m = d rows of S, "one extra bit per dimension" [FQ-TQ QJL section]
    P->S.resize((size_t)d * d);
    sign_fill(seed, 1, (long)d * d, P->S.data());
    P->vbits = bits;
    P->kbits = (key_mode == 0) ? bits - 1 : bits;
    P->beta = beta;
    P->dense3 = dense3;
    P->cv.resize(1 << P->vbits);
    P->tv.resize((1 << P->vbits) - 1);
    P->ck.resize(1 << P->kbits);
    P->tk.resize((1 << P->kbits) - 1);
    if (beta) {
        lloyd_max_beta(d, P->vbits, P->cv.data(), P->tv.data());
        lloyd_max_beta(d, P->kbits, P->ck.data(), P->tk.data());
    } else {
        lloyd_max_gaussian(P->vbits, P->cv.data(), P->tv.data());
        lloyd_max_gaussian(P->kbits, P->ck.data(), P->tk.data());
    }
    return P;
}
void orc_destroy(void* h) { delete (Params*)h; }

void orc_get_rotation(void* h, double* R) {
    Params* P = (Params*)h;
    std::memcpy(R, P->R.data(), sizeof(double) * P->R.size());
}
void orc_get_S(void* h, int8_t* S) {
    Params* P = (Params*)h;
    std::memcpy(S, P->S.data(), P->S.size());
}
int orc_get_hadamard_signs(void* h, int8_t* D) {
    Params* P = (Params*)h;
    if (P->rot != 1) return -1;
    std::memcpy(D, P->D.data(), P->D.size());
    return 0;
}
// kind 0 = key codebook, 1 = value codebook; returns the number of levels
int orc_get_codebook(void* h, int kind, double* c, double* t) {
    Params* P = (Params*)h;
    const std::vector<double>& cc = kind == 1 ? P->cv : P->ck;
    const std::vector<double>& tt = kind == 1 ? P->tv : P->tk;
    std::memcpy(c, cc.data(), sizeof(double) * cc.size());
    std::memcpy(t, tt.data(), sizeof(double) * tt.size());
    return (int)cc.size();
}
long orc_chunk_bytes(void* h, int kind) { return (long)chunk_bytes(*(Params*)h, kind); }
int orc_code_bits(void* h, int kind) {
    Params* P = (Params*)h;
    return kind == 1 ? P->vbits : P->kbits;
}

// ---- compress / decompress of unpacked vectors -----------------------------
// x: [N, d] fp64 (the caller widens fp16 exactly).  codes, signs: [N, d] int.
// norms, gammas: [N] fp64 (exact, before the fp32 rounding of the store).
// vdiag, skdiag: optional [N, d] diagnostics (see compress_vector).
void orc_compress_vectors(void* h, int kind, const double* x, long N, int* codes, int* signs,
                          double* norms, double* gammas, double* vdiag, double* skdiag, int nthreads) {
    Params* P = (Params*)h;
    const int d = P->d;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (long i = 0; i < N; ++i) {
        VecOut o = compress_vector(*P, kind, x + i * d, codes + i * d, signs ? signs + i * d : nullptr,
                                   vdiag ? vdiag + i * d : nullptr, skdiag ? skdiag + i * d : nullptr);
        norms[i] = o.norm;
        if (gammas) gammas[i] = o.gamma;
    }
}

void orc_decompress_vectors(void* h, int kind, const int* codes, const int* signs, const double* norms,
                            const double* gammas, long N, double* out, int nthreads) {
    Params* P = (Params*)h;
    const int d = P->d;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (long i = 0; i < N; ++i)
        decompress_vector(*P, kind, codes + i * d, signs ? signs + i * d : nullptr, norms[i],
                          gammas ? gammas[i] : 0.0, out + i * d);
}

// ---- paged cache -------------------------------------------------------------
// x: [T, H, d] fp64.  slot_mapping[t] = block * 16 + offset.  cache:
// [num_blocks, H, chunk_bytes] bytes.  Tokens whose slot is negative are skipped
// (padding).  Returns the number of tokens whose slot was out of range (skipped).
long orc_compress_paged(void* h, int kind, const double* x, int T, int H, const int32_t* slot_mapping,
                        uint8_t* cache, int num_blocks, int nthreads) {
    Params* P = (Params*)h;
    const int d = P->d;
    const size_t cb = chunk_bytes(*P, kind);
    long bad = 0;
    for (int t = 0; t < T; ++t) {
        long s = slot_mapping[t];
        if (s >= (long)num_blocks * 16) ++bad;
    }
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (long v = 0; v < (long)T * H; ++v) {
        const int t = (int)(v / H), hh = (int)(v % H);
        long s = slot_mapping[t];
        if (s < 0 || s >= (long)num_blocks * 16) continue;
        std::vector<int> codes(d), signs(d, 0);
        VecOut o = compress_vector(*P, kind, x + v * d, codes.data(), signs.data(), nullptr, nullptr);
        uint8_t* chunk = cache + ((size_t)(s / 16) * H + hh) * cb;
        write_row(*P, kind, chunk, (int)(s % 16), codes.data(), signs.data(), o.norm, o.gamma);
    }
    return bad;
}

// Read back unpacked fields of T tokens x H heads from a paged cache.
void orc_read_paged(void* h, int kind, const uint8_t* cache, int T, int H, const int32_t* slot_mapping,
                    int* codes, int* signs, double* norms, double* gammas) {
    Params* P = (Params*)h;
    const int d = P->d;
    const size_t cb = chunk_bytes(*P, kind);
    std::vector<int> sg(d);
    for (long v = 0; v < (long)T * H; ++v) {
        const int t = (int)(v / H), hh = (int)(v % H);
        long s = slot_mapping[t];
        const uint8_t* chunk = cache + ((size_t)(s / 16) * H + hh) * cb;
        double n, g;
        read_row(*P, kind, chunk, (int)(s % 16), codes + v * d, signs ? signs + v * d : sg.data(), &n, &g);
        norms[v] = n;
        if (gammas) gammas[v] = g;
    }
}

void orc_decompress_paged(void* h, int kind, const uint8_t* cache, int T, int H, const int32_t* slot_mapping,
                          double* out, int nthreads) {
    Params* P = (Params*)h;
    const int d = P->d;
    const size_t cb = chunk_bytes(*P, kind);
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (long v = 0; v < (long)T * H; ++v) {
        const int t = (int)(v / H), hh = (int)(v % H);
        long s = slot_mapping[t];
        const uint8_t* chunk = cache + ((size_t)(s / 16) * H + hh) * cb;
        std::vector<int> codes(d), signs(d, 0);
        double n, g;
        read_row(*P, kind, chunk, (int)(s % 16), codes.data(), signs.data(), &n, &g);
        decompress_vector(*P, kind, codes.data(), signs.data(), n, g, out + v * d);
    }
}

// ---- decode attention over the paged compressed cache ----------------------
// For each sequence b and query head h (kv head h / G, G = Hq / Hkv, READING:
// consecutive query heads share a kv head), over tokens t < seq_lens[b] found
// through block_table[b, t / 16]:
//   s_t = scale * ( <q, k_hat_t> + gamma_t * sqrt(pi/2)/d * <S q, 2 sigma_t - 1> )
//   p = softmax(s) (max-subtracted), o = sum_t p_t v_hat_t.
// form 0: explicit dequantize-then-dot in the original domain.
// form 1: rotated domain, <q, k_hat> = n/sqrt(d) <R^T q, c[idx]>, o = R sum_t p_t n_t c[idx_t]/sqrt(d).
// Residual window ([TQ-RS] "Couche 5 — Fenêtre résiduelle" and "Couche 7"
// (residual_window=128); the KIVI page's FP16 residual of the most recent tokens):
// the last tail_lens[b] tokens of sequence b are not compressed; their fp16 keys
// and values tail_k / tail_v [B, tail_cap, Hkv, d] join the same softmax with the
// exact score s_u = scale * <q, k_u> and contribute p_u v_u.  READING: the pages
// only name the window and its size, so the plainest reading is one softmax over
// the compressed tokens and the window's tokens together.  tail_k = NULL: no window.
// q: [B, Hq, d] fp64; out: [B, Hq, d] fp64.  Returns 0, or -1 on a block id,
// sequence length or window length that falls outside the cache / table / window.
int orc_decode_window(void* h, const double* q, const uint8_t* kcache, const uint8_t* vcache, int num_blocks,
                      const int32_t* block_table, int max_blocks, const int32_t* seq_lens, int B, int Hq, int Hkv,
                      const double* tail_k, const double* tail_v, const int32_t* tail_lens, int tail_cap,
                      double scale, int form, double* out, int nthreads) {
    Params* P = (Params*)h;
    const int d = P->d;
    const bool prod = P->key_mode == 0;
    const int G = Hq / Hkv;
    const size_t kcb = chunk_bytes(*P, 0), vcb = chunk_bytes(*P, 1);
    const double sd = std::sqrt((double)d);
    const double qjl = std::sqrt(3.14159265358979323846 / 2.0) / d;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > max_blocks * 16) return -1;
        if (tail_k && (tail_lens[b] < 0 || tail_lens[b] > tail_cap)) return -1;
        for (int p = 0; p < (seq_lens[b] + 15) / 16; ++p) {
            int blk = block_table[(size_t)b * max_blocks + p];
            if (blk < 0 || blk >= num_blocks) return -1;
        }
    }
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), hq = (int)(bh % Hq), hk = hq / G;
        const double* qv = q + bh * d;
        double* ov = out + bh * d;
        const int Tn = seq_lens[b];
        const int Un = tail_k ? tail_lens[b] : 0;
        for (int i = 0; i < d; ++i) ov[i] = 0.0;
        if (Tn + Un == 0) continue;   // READING: an empty sequence attends to nothing -> zeros
        std::vector<double> sq(d, 0.0), qr(d, 0.0);
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += (double)P->S[(size_t)j * d + i] * qv[i];
            sq[j] = s;
        }
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += P->R[(size_t)i * d + j] * qv[i];
            qr[j] = s;
        }
        std::vector<double> sc(Tn + Un);
        std::vector<int> codes(d), signs(d, 0);
        std::vector<double> kv(d);
        for (int t = 0; t < Tn; ++t) {
            int blk = block_table[(size_t)b * max_blocks + t / 16];
            const uint8_t* chunk = kcache + ((size_t)blk * Hkv + hk) * kcb;
            double n, g;
            read_row(*P, 0, chunk, t % 16, codes.data(), signs.data(), &n, &g);
            double dot = 0.0;
            if (form == 0) {
                decompress_vector(*P, 0, codes.data(), signs.data(), n, 0.0, kv.data());  // k_hat only
                for (int i = 0; i < d; ++i) dot += qv[i] * kv[i];
            } else {
                for (int j = 0; j < d; ++j) dot += qr[j] * P->ck[codes[j]];
                dot *= n / sd;
            }
            if (prod) {
                double sg = 0.0;
                for (int j = 0; j < d; ++j) sg += sq[j] * (2.0 * signs[j] - 1.0);
                dot += g * qjl * sg;
            }
            sc[t] = scale * dot;
        }
        // the window's tokens: exact fp16 keys (widened), exact scores
        for (int u = 0; u < Un; ++u) {
            const double* ku = tail_k + (((size_t)b * tail_cap + u) * Hkv + hk) * d;
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qv[i] * ku[i];
            sc[Tn + u] = scale * dot;
        }
        double m = sc[0];
        for (int t = 1; t < Tn + Un; ++t)
            if (sc[t] > m) m = sc[t];
        double den = 0.0;
        for (int t = 0; t < Tn + Un; ++t) {
            sc[t] = std::exp(sc[t] - m);
            den += sc[t];
        }
        std::vector<double> acc(d, 0.0);
        for (int t = 0; t < Tn; ++t) {
            int blk = block_table[(size_t)b * max_blocks + t / 16];
            const uint8_t* chunk = vcache + ((size_t)blk * Hkv + hk) * vcb;
            double n, g;
            read_row(*P, 1, chunk, t % 16, codes.data(), signs.data(), &n, &g);
            const double p = sc[t] / den;
            if (form == 0) {
                decompress_vector(*P, 1, codes.data(), nullptr, n, 0.0, kv.data());
                for (int i = 0; i < d; ++i) ov[i] += p * kv[i];
            } else {
                for (int j = 0; j < d; ++j) acc[j] += p * n * P->cv[codes[j]] / sd;
            }
        }
        if (form == 1)
            for (int i = 0; i < d; ++i) {
                double s = 0.0;
                for (int j = 0; j < d; ++j) s += P->R[(size_t)i * d + j] * acc[j];
                ov[i] = s;
            }
        for (int u = 0; u < Un; ++u) {
            const double* vu = tail_v + (((size_t)b * tail_cap + u) * Hkv + hk) * d;
            const double p = sc[Tn + u] / den;
            for (int i = 0; i < d; ++i) ov[i] += p * vu[i];
        }
    }
    return 0;
}

int orc_decode(void* h, const double* q, const uint8_t* kcache, const uint8_t* vcache, int num_blocks,
               const int32_t* block_table, int max_blocks, const int32_t* seq_lens, int B, int Hq, int Hkv,
               double scale, int form, double* out, int nthreads) {
    return orc_decode_window(h, q, kcache, vcache, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv,
                             nullptr, nullptr, nullptr, 0, scale, form, out, nthreads);
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

}  // extern "C"
