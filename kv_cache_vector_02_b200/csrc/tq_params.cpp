// Host-side parameter generation for libtq (runs once, in tq_init).
//
// [FQ-TQ] = "FlashQuant：生产级KV缓存压缩方案，让大模型推理显存占用降低7.5倍",
//           sections "TurboQuant" (steps 2-3), "QJL校正" (S), "架构设计"
//           (Codebook: Lloyd-Max; Rotation: Haar QR).
// [TQ-RS] = "TurboQuant : compresser le KV-cache des LLM par 7x ...", "Couche 1"
//           (randomized Walsh-Hadamard).
//
// The random streams follow one fixed definition (SplitMix64, Steele/Lea/Flood
// 2014; stream (seed, tag) starts at state seed + tag * 2^48; uniform = top 53
// bits centred in their cell; normals by Box-Muller, both outputs in order;
// a sign is -1 when the top bit of a word is set).  Everything here is host
// C++ in fp64.
#include "tq_internal.h"

#include <cmath>
#include <cstring>
#include <vector>

namespace tq {

namespace {

class SplitMix64 {
  public:
    SplitMix64(uint64_t seed, uint64_t tag) : s_(seed + (tag << 48)) {}
    uint64_t operator()() {
        s_ += 0x9E3779B97F4A7C15ull;
        uint64_t z = s_;
        z ^= z >> 30;
        z *= 0xBF58476D1CE4E5B9ull;
        z ^= z >> 27;
        z *= 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }

  private:
    uint64_t s_;
};

double open_uniform(SplitMix64& g) {
    const double scale = 1.0 / 9007199254740992.0;  // 2^-53
    return (static_cast<double>(g() >> 11) + 0.5) * scale;
}

std::vector<double> normals(uint64_t seed, uint64_t tag, size_t n) {
    SplitMix64 g(seed, tag);
    std::vector<double> z(n);
    const double tau = 2.0 * M_PI;
    size_t i = 0;
    while (i < n) {
        const double a = open_uniform(g);
        const double b = open_uniform(g);
        const double rho = std::sqrt(-2.0 * std::log(a));
        z[i++] = rho * std::cos(tau * b);
        if (i < n) z[i++] = rho * std::sin(tau * b);
    }
    return z;
}

std::vector<int8_t> rademacher(uint64_t seed, uint64_t tag, size_t n) {
    SplitMix64 g(seed, tag);
    std::vector<int8_t> s(n);
    for (size_t i = 0; i < n; ++i) s[i] = (g() >> 63) ? int8_t(-1) : int8_t(1);
    return s;
}

// Q factor of G (row-major d x d) by classical Gram-Schmidt applied twice per
// column ("CGS2").  Gram-Schmidt yields a triangular factor with positive
// diagonal, so Q is the unique such factor: the Haar-distributed rotation.
std::vector<double> gram_schmidt_q(const std::vector<double>& G, int d) {
    std::vector<double> Q(size_t(d) * d, 0.0);  // column-major working copy: Q[c*d + r]
    std::vector<double> v(d);
    for (int c = 0; c < d; ++c) {
        for (int r = 0; r < d; ++r) v[r] = G[size_t(r) * d + c];
        for (int pass = 0; pass < 2; ++pass) {
            for (int p = 0; p < c; ++p) {
                const double* qp = &Q[size_t(p) * d];
                double proj = 0.0;
                for (int r = 0; r < d; ++r) proj += qp[r] * v[r];
                for (int r = 0; r < d; ++r) v[r] -= proj * qp[r];
            }
        }
        double nn = 0.0;
        for (int r = 0; r < d; ++r) nn += v[r] * v[r];
        const double inv = 1.0 / std::sqrt(nn);
        for (int r = 0; r < d; ++r) Q[size_t(c) * d + r] = v[r] * inv;
    }
    std::vector<double> R(size_t(d) * d);
    for (int r = 0; r < d; ++r)
        for (int c = 0; c < d; ++c) R[size_t(r) * d + c] = Q[size_t(c) * d + r];
    return R;
}

// Sylvester-ordered Hadamard entry H[i][j] = (-1)^popcount(i & j).
inline double hadamard_entry(int i, int j) { return (__builtin_popcount(unsigned(i & j)) & 1) ? -1.0 : 1.0; }

// Upper-tail probability of the unit normal, Q(x) = P(X > x).
inline double upper_tail(double x) { return 0.5 * std::erfc(x / M_SQRT2); }
inline double density(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); }

// Gaussian Lloyd-Max codebook with L = 2^bits levels, solved on the positive
// half (the law is symmetric, so c_{L-1-j} = -c_j and 0 is a boundary):
//   positive levels a_1 < ... < a_m (m = L/2), boundaries 0 = e_0 < e_1 < ... < e_m = inf
//   a_k = (phi(e_{k-1}) - phi(e_k)) / (Q(e_{k-1}) - Q(e_k)),  e_k = (a_k + a_{k+1}) / 2.
void gaussian_lloyd_max(int bits, std::vector<double>& levels, std::vector<double>& bounds) {
    const int L = 1 << bits, m = L / 2;
    std::vector<double> a(m), e(m + 1);
    for (int k = 0; k < m; ++k) a[k] = 3.0 * (k + 0.5) / m;
    for (int iter = 0; iter < 400000; ++iter) {
        e[0] = 0.0;
        for (int k = 1; k < m; ++k) e[k] = 0.5 * (a[k - 1] + a[k]);
        double delta = 0.0;
        for (int k = 0; k < m; ++k) {
            const double lo = e[k];
            const bool last = (k == m - 1);
            const double num = density(lo) - (last ? 0.0 : density(e[k + 1]));
            const double den = upper_tail(lo) - (last ? 0.0 : upper_tail(e[k + 1]));
            const double nv = num / den;
            delta = std::fmax(delta, std::fabs(nv - a[k]));
            a[k] = nv;
        }
        if (delta < 1e-16) break;
    }
    levels.assign(L, 0.0);
    for (int k = 0; k < m; ++k) {
        levels[m + k] = a[k];
        levels[m - 1 - k] = -a[k];
    }
    bounds.assign(L - 1, 0.0);
    for (int j = 0; j + 1 < L; ++j) bounds[j] = 0.5 * (levels[j] + levels[j + 1]);
    bounds[m - 1] = 0.0;
}

// Exact-d Lloyd-Max codebook ([TQ-RS] "Étape 2" / "Couche 2": the rotated
// coordinate of a unit vector follows the spherical Beta law).  The quantized
// value is v = sqrt(d) cos(theta), where the angle theta of a uniform unit vector
// to an axis has density proportional to sin^n(theta), n = d - 2, on (0, pi).
// With J(alpha) = int_0^alpha sin^n, by the reduction formula
//   J_k(alpha) = -sin^(k-1)(alpha) cos(alpha) / k + (k-1)/k J_(k-2)(alpha),
//   P(v > x)   = J(acos(x / sqrt(d))) / J(pi),
//   E[v; v > x] = sqrt(d) sin^(n+1)(acos(x / sqrt(d))) / ((n+1) J(pi)).
// (The recursion loses relative accuracy in the far tail, beyond the largest
// boundary a 4-bit codebook has; the last cell's mass is dominated by its start.)
// Solved on the positive half like the Gaussian codebook.
double sin_power_integral(int n, double alpha) {
    const double s = std::sin(alpha), c = std::cos(alpha);
    double j = (n % 2 == 0) ? alpha : 1.0 - c;
    double sp = (n % 2 == 0) ? s : s * s;  // sin^(k-1) for the first k
    for (int k = (n % 2 == 0) ? 2 : 3; k <= n; k += 2) {
        j = -sp * c / k + double(k - 1) / k * j;
        sp *= s * s;
    }
    return j;
}

void sphere_lloyd_max(int d, int bits, std::vector<double>& levels, std::vector<double>& bounds) {
    const int L = 1 << bits, m = L / 2, n = d - 2;
    const double rd = std::sqrt(double(d)), total = sin_power_integral(n, M_PI);
    auto tail = [&](double x) { return sin_power_integral(n, std::acos(std::fmin(x / rd, 1.0))) / total; };
    auto tail_moment = [&](double x) {
        const double th = std::acos(std::fmin(x / rd, 1.0));
        return rd * std::pow(std::sin(th), n + 1) / ((n + 1) * total);
    };
    std::vector<double> a(m), e(m + 1);
    for (int k = 0; k < m; ++k) a[k] = 3.0 * (k + 0.5) / m;
    for (int iter = 0; iter < 400000; ++iter) {
        e[0] = 0.0;
        for (int k = 1; k < m; ++k) e[k] = 0.5 * (a[k - 1] + a[k]);
        double delta = 0.0;
        for (int k = 0; k < m; ++k) {
            const bool last = (k == m - 1);
            const double num = tail_moment(e[k]) - (last ? 0.0 : tail_moment(e[k + 1]));
            const double den = tail(e[k]) - (last ? 0.0 : tail(e[k + 1]));
            const double nv = num / den;
            delta = std::fmax(delta, std::fabs(nv - a[k]));
            a[k] = nv;
        }
        if (delta < 1e-16) break;
    }
    levels.assign(L, 0.0);
    for (int k = 0; k < m; ++k) {
        levels[m + k] = a[k];
        levels[m - 1 - k] = -a[k];
    }
    bounds.assign(L - 1, 0.0);
    for (int j = 0; j + 1 < L; ++j) bounds[j] = 0.5 * (levels[j] + levels[j + 1]);
    bounds[m - 1] = 0.0;
}

}  // namespace

HostParams make_host_params(int d, int bits, uint64_t seed, int rotation, int key_mode, int flags) {
    HostParams P;
    P.d = d;
    P.bits = bits;
    P.rotation = rotation;
    P.key_mode = key_mode;
    P.vbits = bits;
    P.kbits = (key_mode == 0) ? bits - 1 : bits;
    if (rotation == 0) {
        P.R = gram_schmidt_q(normals(seed, 0, size_t(d) * d), d);
    } else {
        P.hsigns = rademacher(seed, 2, size_t(d));
        P.R.resize(size_t(d) * d);
        const double s = 1.0 / std::sqrt(double(d));
        for (int i = 0; i < d; ++i)  // R = D H / sqrt(d)
            for (int j = 0; j < d; ++j) P.R[size_t(i) * d + j] = P.hsigns[i] * hadamard_entry(i, j) * s;
    }
    P.S = rademacher(seed, 1, size_t(d) * d);
    P.flags = flags;
    if (flags & TQ_FLAG_SPHERE_CODEBOOK) {
        sphere_lloyd_max(d, P.vbits, P.cv, P.tv);
        sphere_lloyd_max(d, P.kbits, P.ck, P.tk);
    } else {
        gaussian_lloyd_max(P.vbits, P.cv, P.tv);
        gaussian_lloyd_max(P.kbits, P.ck, P.tk);
    }
    // M = S R: the QJL sketch taken in the rotated domain, S r = S R (R^T r).
    P.M.assign(size_t(d) * d, 0.0);
    for (int j = 0; j < d; ++j)
        for (int k = 0; k < d; ++k) {
            const double sjk = P.S[size_t(j) * d + k];
            for (int i = 0; i < d; ++i) P.M[size_t(j) * d + i] += sjk * P.R[size_t(k) * d + i];
        }
    return P;
}

}  // namespace tq
