// oracle.cc -- plain, slow, single-threaded fp64 CPU oracle for rotated-token
// KV-cache quantization (TurboQuant form, with the NSN front end).
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
// calls this file; only tests/, __graft_entry__.smoke() and bench.py's CPU
// baseline leg do.  It shares no code, header, table or constant generator
// with the CUDA library: every step is written out again here from the
// method's definition, in fp64, in the order the sources describe it.
//
// Sources (web pages, cited by title and section):
//   [TQ]  "O Que E TurboQuant? A Inovadora Compressao de IA do Google para
//         Cache KV 6x Menor" -- sections "Estagio 1: Rotacao Aleatoria +
//         Compressao PolarQuant" and "Estagio 2: Correcao Residual QJL";
//         "Como Implementar" (precomputed Lloyd-Max codebooks, queries
//         rotated once, logits straight from the indices).
//   [PQ]  "PolarQuant: Optimal Gaussian Weight Quantization via Hadamard
//         Rotation for LLM Compression" -- Resumo Tecnico, section 2
//         "Metodologia" (block normalisation, Walsh-Hadamard rotation,
//         scaling to unit variance, Gaussian Lloyd-Max centroids,
//         dequantisation as the exact inverse).
//   [NSN] "NSNQuant: A Double Normalization Approach for Calibration-Free
//         Low-Bit Vector Quantization of KV Cache" -- Resumo Tecnico,
//         sections 1 (Normalize-Shift-Normalize), 2 (Hadamard / RHT) and
//         4 (residual window; attention from the byproducts).
//
// Where the pages leave a step open, the reading taken is the one listed in
// the repository's design notes (readings table); each function says which.
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -o liboracle.so oracle.cc
// (no -ffast-math: IEEE fp64 semantics are part of the contract).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

const double kPi = 3.14159265358979323846264338327950288;

// Sylvester-ordered, unnormalised Walsh-Hadamard entry:
// H[i][j] = (-1)^popcount(i & j)   ([PQ] sec. 2 "Rotacao de Hadamard").
inline double hadamard_entry(int i, int j) {
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
}

// Standard normal density and distribution function.
inline double normal_pdf(double x) {
    if (std::isinf(x)) return 0.0;
    return std::exp(-0.5 * x * x) / std::sqrt(2.0 * kPi);
}
inline double normal_cdf(double x) {
    if (x == INFINITY) return 1.0;
    if (x == -INFINITY) return 0.0;
    return 0.5 * std::erfc(-x / std::sqrt(2.0));
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Counter-based random numbers (the pages draw random signs and a Gaussian
// projection but do not say how; reading: SplitMix64).
//
// SplitMix64 as published by Steele, Lea and Flood ("Fast splittable
// pseudorandom number generators", OOPSLA 2014) in Vigna's reference form:
// the state advances by the golden-ratio increment before each output, so
// output i (0-based) of a stream seeded with s is mix(s + (i+1)*gamma).
// ---------------------------------------------------------------------------
uint64_t orc_splitmix64(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

// Rademacher signs of the randomized Hadamard transform ([NSN] sec. 2 RHT;
// [TQ] Stage 1.1 "rotacao ortogonal aleatoria", taken as the RHT):
// delta_j = +1 when the top bit of output j of the stream is 0, else -1.
void orc_rademacher_signs(int d, uint64_t seed, int8_t* delta) {
    for (int j = 0; j < d; ++j)
        delta[j] = (orc_splitmix64(seed, (uint64_t)j) >> 63) ? (int8_t)-1 : (int8_t)1;
}

// IEEE binary16 round-to-nearest-even of a double, written out from the
// binary16 format definition (sign, 5-bit exponent bias 15, 10-bit fraction,
// subnormals, infinity).  Returns the 16 bit pattern.
uint16_t orc_double_to_half(double x) {
    uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
    if (std::isnan(x)) return (uint16_t)(sign | 0x7E00u);
    double a = std::fabs(x);
    if (std::isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a < std::ldexp(1.0, -14)) {
        // subnormal range: a = k * 2^-24, k in [0, 1024]; k == 1024 is the
        // smallest normal (0x0400), which the bit pattern below also gives.
        double k = std::nearbyint(std::ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)k);
    }
    int e = 0;
    double f = std::frexp(a, &e);               // a = f * 2^e, f in [0.5, 1)
    double k = std::nearbyint(std::ldexp(f, 11));  // significand in [1024, 2048]
    int E = e - 1;                              // a = (k / 1024) * 2^E
    if (k == 2048.0) { k = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)k - 1024));
}

double orc_half_to_double(uint16_t h) {
    double s = (h & 0x8000u) ? -1.0 : 1.0;
    int E = (h >> 10) & 0x1F;
    int F = h & 0x3FF;
    if (E == 0) return s * std::ldexp((double)F, -24);
    if (E == 31) return F ? NAN : s * INFINITY;
    return s * std::ldexp(1024.0 + F, E - 25);
}

// Gaussian projection S (rows x cols, row-major) of the QJL residual sketch
// ([TQ] Stage 2).  Element k (row-major index) uses outputs 2k and 2k+1 of
// the stream: u1 = (top 53 bits of o_2k + 1) * 2^-53 in (0, 1],
// u2 = (top 53 bits of o_2k+1) * 2^-53 in [0, 1), and the cosine branch of
// the Box-Muller transform, g = sqrt(-2 ln u1) cos(2 pi u2).  The value is
// then rounded to binary16; the rounded value IS the matrix S of the method
// (reading: S is held in fp16 so that it is an exact tensor-core operand).
// Writes the fp16 bit patterns and, optionally, the unrounded draws.
void orc_gaussian_fp16(int rows, int cols, uint64_t seed, uint16_t* s_half, double* draws) {
    for (int64_t k = 0; k < (int64_t)rows * cols; ++k) {
        uint64_t o1 = orc_splitmix64(seed, (uint64_t)(2 * k));
        uint64_t o2 = orc_splitmix64(seed, (uint64_t)(2 * k + 1));
        double u1 = (double)((o1 >> 11) + 1) * std::ldexp(1.0, -53);
        double u2 = (double)(o2 >> 11) * std::ldexp(1.0, -53);
        double g = std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * kPi * u2);
        if (draws) draws[k] = g;
        s_half[k] = orc_double_to_half(g);
    }
}

// ---------------------------------------------------------------------------
// Lloyd-Max scalar quantizer for a standard Gaussian with L = 2^b levels
// ([PQ] sec. 2 "Escalonamento e Quantizacao": Lloyd-Max centroids, optimal
// for the Gaussian; [TQ] "pre-calcule codebooks Lloyd-Max" per bit-width).
// Lloyd's iteration: thresholds are the midpoints of adjacent centroids,
// centroids are the conditional means of N(0,1) over their cells,
//   c_k = (phi(t_k) - phi(t_{k+1})) / (Phi(t_{k+1}) - Phi(t_k)),
// with t_0 = -inf, t_L = +inf, repeated until no centroid moves by more than
// `tol` or `max_iter` steps have run.  Writes L centroids (ascending), L-1
// interior thresholds and the mean squared error of the final codebook
// (cell by cell in closed form).  Returns the number of steps taken.
// ---------------------------------------------------------------------------
int orc_lloyd_max_gaussian(int b, double* centroid, double* threshold, double* mse,
                           int max_iter, double tol) {
    const int L = 1 << b;
    std::vector<double> c(L), t(L + 1), cn(L);
    for (int k = 0; k < L; ++k) c[k] = -2.0 + 4.0 * (k + 0.5) / L;
    int it = 0;
    for (; it < max_iter; ++it) {
        t[0] = -INFINITY;
        t[L] = INFINITY;
        for (int k = 1; k < L; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
        double move = 0.0;
        for (int k = 0; k < L; ++k) {
            double p = normal_cdf(t[k + 1]) - normal_cdf(t[k]);
            cn[k] = (normal_pdf(t[k]) - normal_pdf(t[k + 1])) / p;
            move = std::fmax(move, std::fabs(cn[k] - c[k]));
        }
        c = cn;
        if (move <= tol) { ++it; break; }
    }
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int k = 1; k < L; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
    // Cell error: int_a^b (x-c)^2 phi = p(1+c^2) + a phi(a) - b phi(b) - 2c(phi(a)-phi(b)).
    double D = 0.0;
    for (int k = 0; k < L; ++k) {
        double a = t[k], bb = t[k + 1];
        double p = normal_cdf(bb) - normal_cdf(a);
        double apa = std::isinf(a) ? 0.0 : a * normal_pdf(a);
        double bpb = std::isinf(bb) ? 0.0 : bb * normal_pdf(bb);
        D += p * (1.0 + c[k] * c[k]) + apa - bpb - 2.0 * c[k] * (normal_pdf(a) - normal_pdf(bb));
    }
    for (int k = 0; k < L; ++k) centroid[k] = c[k];
    for (int k = 1; k < L; ++k) threshold[k - 1] = t[k];
    *mse = D;
    return it;
}

// ---------------------------------------------------------------------------
// Randomized Hadamard rotation of one vector, as a direct matrix product:
// y = H (delta (.) v), O(d^2) on purpose (no butterfly), [NSN] sec. 2,
// [PQ] sec. 2.
// ---------------------------------------------------------------------------
void orc_rht(int d, const int8_t* delta, const double* v, double* y) {
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += hadamard_entry(i, j) * (double)delta[j] * v[j];
        y[i] = s;
    }
}

// QJL residual sketch ([TQ] Stage 2): u = S r, bit_i = [u_i >= 0]
// (reading: one bit per projection row, m rows; sign(0) taken as +).
void orc_qjl_sketch(int m, int d, const double* S, const double* r, uint8_t* bits, double* u_out) {
    for (int i = 0; i < m; ++i) {
        double u = 0.0;
        for (int j = 0; j < d; ++j) u += S[(int64_t)i * d + j] * r[j];
        bits[i] = (u >= 0.0) ? 1 : 0;
        if (u_out) u_out[i] = u;
    }
}

// QJL inner-product estimate of <q, r> from the sketch of r:
// est = sqrt(pi/2)/m * ||r|| * sum_i (S q)_i * (2 bit_i - 1)  ([TQ] Stage 2:
// the 1-bit sketch corrects the inner-product bias; estimator of the
// quantized Johnson-Lindenstrauss transform).
double orc_qjl_estimate(int m, int d, const double* S, const double* q, const uint8_t* bits,
                        double rnorm) {
    double acc = 0.0;
    for (int i = 0; i < m; ++i) {
        double p = 0.0;
        for (int j = 0; j < d; ++j) p += S[(int64_t)i * d + j] * q[j];
        acc += p * (bits[i] ? 1.0 : -1.0);
    }
    return std::sqrt(kPi / 2.0) / m * rnorm * acc;
}

// T independent draws of the QJL estimate of <q, r>: trial k draws its own
// fp16 Gaussian S (m x d) from the stream seeded with seed0 + k, sketches r
// with it and estimates <q, r> from the sketch (used to check that the
// estimator is unbiased, the property [TQ] Stage 2 relies on).
void orc_qjl_trials(int m, int d, const double* q, const double* r, int64_t T, uint64_t seed0,
                    double* est) {
    std::vector<uint16_t> sh((size_t)m * d);
    std::vector<double> S((size_t)m * d);
    std::vector<uint8_t> bits(m);
    double rr = 0.0;
    for (int j = 0; j < d; ++j) rr += r[j] * r[j];
    const double rn = std::sqrt(rr);
    for (int64_t k = 0; k < T; ++k) {
        orc_gaussian_fp16(m, d, seed0 + (uint64_t)k, sh.data(), nullptr);
        for (size_t e = 0; e < sh.size(); ++e) S[e] = orc_half_to_double(sh[e]);
        orc_qjl_sketch(m, d, S.data(), r, bits.data(), nullptr);
        est[k] = orc_qjl_estimate(m, d, S.data(), q, bits.data(), rn);
    }
}

// ---------------------------------------------------------------------------
// Quantize n vectors of dimension d (row-major x), [TQ] Stages 1-2, [PQ] 2:
//   norm  = ||x||
//   z     = H (delta (.) x) / norm          (unit-variance coordinates)
//   code_j = #{k : z_j >= t_k}              (Lloyd-Max cell; ties go up)
//   r     = z - c[code]
//   gamma = ||r||
//   bits  = [S r >= 0]                      (only when use_qjl)
// A zero vector gives all codes 0, all bits 0, norm = gamma = 0.
// Outputs are unpacked: codes[n*d], bits[n*m] (0/1), norm[n], gamma[n];
// z_out[n*d] and u_out[n*m] (nullable) expose the intermediate values for
// the boundary-exclusion rule of the parity tests.
// ---------------------------------------------------------------------------
void orc_quantize(int d, int b, int m, int use_qjl, const int8_t* delta, const double* S,
                  const double* centroid, const double* threshold, const double* x, int64_t n,
                  int32_t* codes, uint8_t* bits, double* norm, double* gamma, double* z_out,
                  double* u_out) {
    const int L = 1 << b;
    std::vector<double> z(d), r(d), u(m > 0 ? m : 1);
    for (int64_t v = 0; v < n; ++v) {
        const double* xv = x + v * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += xv[j] * xv[j];
        double nrm = std::sqrt(ss);
        if (nrm == 0.0) {
            for (int j = 0; j < d; ++j) {
                codes[v * d + j] = 0;
                if (z_out) z_out[v * d + j] = 0.0;
            }
            if (use_qjl)
                for (int i = 0; i < m; ++i) {
                    bits[v * m + i] = 0;
                    if (u_out) u_out[v * m + i] = 0.0;
                }
            norm[v] = 0.0;
            gamma[v] = 0.0;
            continue;
        }
        orc_rht(d, delta, xv, z.data());
        for (int j = 0; j < d; ++j) z[j] /= nrm;
        double rr = 0.0;
        for (int j = 0; j < d; ++j) {
            int code = 0;
            for (int k = 0; k < L - 1; ++k)
                if (z[j] >= threshold[k]) ++code;
            codes[v * d + j] = code;
            r[j] = z[j] - centroid[code];
            rr += r[j] * r[j];
            if (z_out) z_out[v * d + j] = z[j];
        }
        norm[v] = nrm;
        gamma[v] = std::sqrt(rr);
        if (use_qjl) orc_qjl_sketch(m, d, S, r.data(), bits + v * m, u_out ? u_out + v * m : nullptr);
    }
}

// ---------------------------------------------------------------------------
// Explicit dequantisation ([PQ] sec. 2 "Dequantizacao": centroids, inverse
// rotation -- H is its own inverse up to 1/d -- and the stored norm), plus
// the QJL reconstruction of the residual ([TQ] Stage 2):
//   xhat = (norm/d) * delta (.) H (c[code] + sqrt(pi/2)/m * gamma * S^T (2 bits - 1))
// Used only as an independent route for the brute-force attention check.
// ---------------------------------------------------------------------------
void orc_dequantize(int d, int b, int m, int use_qjl, const int8_t* delta, const double* S,
                    const double* centroid, const int32_t* codes, const uint8_t* bits,
                    const double* norm, const double* gamma, int64_t n, double* xhat) {
    (void)b;
    std::vector<double> zh(d), y(d);
    const double kappa = std::sqrt(kPi / 2.0) / (m > 0 ? m : 1);
    for (int64_t v = 0; v < n; ++v) {
        for (int j = 0; j < d; ++j) zh[j] = centroid[codes[v * d + j]];
        if (use_qjl)
            for (int j = 0; j < d; ++j) {
                double s = 0.0;
                for (int i = 0; i < m; ++i)
                    s += S[(int64_t)i * d + j] * (bits[v * m + i] ? 1.0 : -1.0);
                zh[j] += kappa * gamma[v] * s;
            }
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += hadamard_entry(i, j) * zh[j];
            y[i] = s;
        }
        for (int i = 0; i < d; ++i) xhat[v * d + i] = norm[v] / d * (double)delta[i] * y[i];
    }
}

// ---------------------------------------------------------------------------
// Decode attention over one KV head's key and value caches for G query vectors
// ([TQ] "Como Implementar": queries are rotated once and the attention
// logits come straight from the stored indices; [PQ] sec. 2 dequantisation
// algebra moved to the query side).  Single pass, max-subtracted softmax,
// no splitting:
//   q'   = H (delta (.) q)             p = S q'
//   l_t  = scale * (n_t/d) * ( sum_j q'_j c[code_tj]
//                              + sqrt(pi/2)/m * gamma_t * sum_i p_i (2 bit_ti - 1) )   (keys)
//   w_t  = exp(l_t - max l)            Lsum = sum_t w_t
//   A_j  = sum_t w_t n_t c[code_tj]    B_i = sum_t w_t n_t gamma_t (2 bit_ti - 1)      (values)
//   out  = 1/(d Lsum) * delta (.) H (A + sqrt(pi/2)/m * S^T B)
// norm/gamma are the values the cache stores (fp16, widened).  T == 0 gives
// an all-zero output.  logits (G x T) is nullable.
// ---------------------------------------------------------------------------
void orc_decode_attend(int d, int b, int m, int use_qjl, const int8_t* delta, const double* S,
                       const double* centroid, const double* q, int G, const int32_t* kcodes,
                       const uint8_t* kbits, const double* knorm, const double* kgamma,
                       const int32_t* vcodes, const uint8_t* vbits, const double* vnorm,
                       const double* vgamma, int64_t T, double scale, double* logits, double* out) {
    (void)b;
    const double kappa = std::sqrt(kPi / 2.0) / (m > 0 ? m : 1);
    std::vector<double> qr(d), p(m > 0 ? m : 1), l(T > 0 ? T : 1), A(d), B(m > 0 ? m : 1), v(d), y(d);
    for (int g = 0; g < G; ++g) {
        if (T == 0) {
            for (int j = 0; j < d; ++j) out[(int64_t)g * d + j] = 0.0;
            continue;
        }
        orc_rht(d, delta, q + (int64_t)g * d, qr.data());
        if (use_qjl)
            for (int i = 0; i < m; ++i) {
                double s = 0.0;
                for (int j = 0; j < d; ++j) s += S[(int64_t)i * d + j] * qr[j];
                p[i] = s;
            }
        double M = -INFINITY;
        for (int64_t t = 0; t < T; ++t) {
            double dot = 0.0;
            for (int j = 0; j < d; ++j) dot += qr[j] * centroid[kcodes[t * d + j]];
            if (use_qjl) {
                double s = 0.0;
                for (int i = 0; i < m; ++i) s += p[i] * (kbits[t * m + i] ? 1.0 : -1.0);
                dot += kappa * kgamma[t] * s;
            }
            l[t] = scale * (knorm[t] / d) * dot;
            if (logits) logits[(int64_t)g * T + t] = l[t];
            M = std::fmax(M, l[t]);
        }
        double Lsum = 0.0;
        for (int j = 0; j < d; ++j) A[j] = 0.0;
        for (int i = 0; i < m; ++i) B[i] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double w = std::exp(l[t] - M);
            Lsum += w;
            for (int j = 0; j < d; ++j) A[j] += w * vnorm[t] * centroid[vcodes[t * d + j]];
            if (use_qjl)
                for (int i = 0; i < m; ++i)
                    B[i] += w * vnorm[t] * vgamma[t] * (vbits[t * m + i] ? 1.0 : -1.0);
        }
        for (int j = 0; j < d; ++j) {
            double s = A[j];
            if (use_qjl) {
                double st = 0.0;
                for (int i = 0; i < m; ++i) st += S[(int64_t)i * d + j] * B[i];
                s += kappa * st;
            }
            v[j] = s;
        }
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int j = 0; j < d; ++j) s += hadamard_entry(i, j) * v[j];
            y[i] = s;
        }
        for (int i = 0; i < d; ++i) out[(int64_t)g * d + i] = (double)delta[i] * y[i] / (d * Lsum);
    }
}

// ---------------------------------------------------------------------------
// NSN front end ([NSN] sec. 1 Normalize-Shift-Normalize, sec. 4 residual
// flush granularity), on n_tok tokens of one head, blocks of `blk` tokens:
//   u_t   = sqrt(d) x_t / ||x_t||            (zero token: u_t = 0)
//   o     = mean over the block of u_t, per channel   -> rounded to fp16
//   w_t   = u_t - fp16(o)                    (the stored mean is subtracted,
//                                             so decode sees what was used)
//   then the quantizer above on w_t without the QJL stage; the token keeps
//   fp16 ||x_t|| (s1 = ||x||/sqrt d) and fp16 ||w_t|| (s2 = ||w||/sqrt d).
// mean_in (nullable, (n_tok/blk) x d fp16 patterns) replaces the rounding of
// o by a caller-chosen neighbour; mean_f64 (nullable) returns the unrounded
// block means.  Outputs: codes[n_tok*d], norm_x[n_tok], norm_w[n_tok],
// mean_half[(n_tok/blk)*d], z_out (nullable).
// ---------------------------------------------------------------------------
void orc_nsn_quantize(int d, int b, int blk, const int8_t* delta, const double* centroid,
                      const double* threshold, const double* x, int64_t n_tok,
                      const uint16_t* mean_in, int32_t* codes, double* norm_x, double* norm_w,
                      uint16_t* mean_half, double* mean_f64, double* z_out) {
    std::vector<double> u((size_t)blk * d), o(d), w(d), gdummy(1);
    const double sqd = std::sqrt((double)d);
    for (int64_t b0 = 0; b0 < n_tok; b0 += blk) {
        int64_t blk_id = b0 / blk;
        for (int t = 0; t < blk; ++t) {
            const double* xv = x + (b0 + t) * d;
            double ss = 0.0;
            for (int j = 0; j < d; ++j) ss += xv[j] * xv[j];
            double nx = std::sqrt(ss);
            norm_x[b0 + t] = nx;
            for (int j = 0; j < d; ++j) u[(size_t)t * d + j] = (nx == 0.0) ? 0.0 : sqd * xv[j] / nx;
        }
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int t = 0; t < blk; ++t) s += u[(size_t)t * d + j];
            o[j] = s / blk;
            if (mean_f64) mean_f64[blk_id * d + j] = o[j];
            uint16_t h = mean_in ? mean_in[blk_id * d + j] : orc_double_to_half(o[j]);
            mean_half[blk_id * d + j] = h;
        }
        for (int t = 0; t < blk; ++t) {
            for (int j = 0; j < d; ++j)
                w[j] = u[(size_t)t * d + j] - orc_half_to_double(mean_half[blk_id * d + j]);
            double nw = 0.0, gam = 0.0;
            orc_quantize(d, b, 0, 0, delta, nullptr, centroid, threshold, w.data(), 1,
                         codes + (b0 + t) * d, nullptr, &nw, &gam,
                         z_out ? z_out + (b0 + t) * d : nullptr, nullptr);
            norm_w[b0 + t] = nw;
        }
    }
}

// ---------------------------------------------------------------------------
// NSN front end with double quantization of its side data ([NSN] sec. 3,
// "Double Quantization": the NSN parameters -- the mean o and the scale s1 --
// are themselves quantized to 4 bits).  The pages give no format; the reading
// (recorded with the design notes) is, per block of `blk` tokens of one head:
//   s1:  4-bit linear codes of the token norms on the block's own step
//        nstep = fp16(max_t ||x_t|| / 15):  q = 0 for a zero token, else
//        q = clamp(rint(||x|| / nstep), 1, 15);  n1 = q * nstep  (exact);
//   u_t = sqrt(d) x_t / n1_t              (0 for q = 0)
//   o   = mean over the block of u_t, per channel;
//   o:   4-bit linear codes on [lo, lo + 15 step] with lo = fp16(min_j o_j),
//        step = fp16((max_j o_j - min_j o_j) / 15):
//        q_j = clamp(rint((o_j - lo) / step), 0, 15)  (0 when step = 0),
//        o_hat_j = fp32(lo + step q_j)   (the exact sum rounded once to fp32)
//   w_t = u_t - o_hat, quantized like the plain NSN front end (no QJL);
//   stored: codes, fp16 ||w_t||, and one side record per block:
//     bytes [0,2) fp16 lo, [2,4) fp16 step, [4,6) fp16 nstep, [6,8) zero,
//     [8, 8 + d/2) o codes (byte i: channel 2i low nibble, 2i+1 high),
//     [8 + d/2, 8 + d/2 + blk/2) norm codes (byte i: token 2i low, 2i+1 high),
//     zero padding to a multiple of 16 bytes (rec_bytes).
// The stored values are the ones the transform used, so x_t = n1_t / sqrt(d)
// (w_t + o_hat) exactly before w_t is coded.  side_in (nullable) replaces
// parts of this function's side records by given ones, so that the rest can
// be recomputed for a record another implementation wrote: side_parts bit 0
// takes the norm step and codes from side_in, bit 1 the mean offset, step
// and codes.
// Outputs: codes[n_tok*d], norm_w[n_tok], side_out[(n_tok/blk)*rec_bytes],
// n1[n_tok], o_hat[(n_tok/blk)*d], o_f64[(n_tok/blk)*d] (unquantized
// means), norm_x[n_tok] (unquantized norms), z_out (nullable).
// ---------------------------------------------------------------------------
int orc_nsn_dq_rec_bytes(int d, int blk) { return (8 + d / 2 + blk / 2 + 15) / 16 * 16; }

void orc_nsn_dq_quantize(int d, int b, int blk, const int8_t* delta, const double* centroid,
                         const double* threshold, const double* x, int64_t n_tok, const uint8_t* side_in,
                         int side_parts, int32_t* codes, double* norm_w, uint8_t* side_out, double* n1, double* o_hat,
                         double* o_f64, double* norm_x, double* z_out) {
    const int R = orc_nsn_dq_rec_bytes(d, blk);
    const bool in_n = side_in && (side_parts & 1), in_o = side_in && (side_parts & 2);
    std::vector<double> u((size_t)blk * d), o(d), w(d);
    const double sqd = std::sqrt((double)d);
    for (int64_t b0 = 0; b0 < n_tok; b0 += blk) {
        const int64_t bi = b0 / blk;
        uint8_t* rec = side_out + bi * R;
        for (int e = 0; e < R; ++e) rec[e] = 0;
        // token norms and their 4-bit codes
        double mx = 0.0;
        for (int t = 0; t < blk; ++t) {
            const double* xv = x + (b0 + t) * d;
            double ss = 0.0;
            for (int j = 0; j < d; ++j) ss += xv[j] * xv[j];
            norm_x[b0 + t] = std::sqrt(ss);
            mx = std::fmax(mx, norm_x[b0 + t]);
        }
        uint16_t nstep16 = orc_double_to_half(mx / 15.0);
        if (in_n) nstep16 = (uint16_t)(side_in[bi * R + 4] | (side_in[bi * R + 5] << 8));
        const double nstep = orc_half_to_double(nstep16);
        rec[4] = (uint8_t)(nstep16 & 0xFF);
        rec[5] = (uint8_t)(nstep16 >> 8);
        for (int t = 0; t < blk; ++t) {
            int q;
            if (in_n) {
                const uint8_t by = side_in[bi * R + 8 + d / 2 + t / 2];
                q = (t & 1) ? (by >> 4) : (by & 15);
            } else if (norm_x[b0 + t] == 0.0 || nstep == 0.0) {
                q = 0;
            } else {
                q = (int)std::nearbyint(norm_x[b0 + t] / nstep);
                q = q < 1 ? 1 : (q > 15 ? 15 : q);
            }
            rec[8 + d / 2 + t / 2] |= (uint8_t)(q << ((t & 1) * 4));
            n1[b0 + t] = q * nstep;
            const double* xv = x + (b0 + t) * d;
            for (int j = 0; j < d; ++j) u[(size_t)t * d + j] = (q == 0) ? 0.0 : sqd * xv[j] / n1[b0 + t];
        }
        // channel means and their 4-bit codes
        double lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int t = 0; t < blk; ++t) s += u[(size_t)t * d + j];
            o[j] = s / blk;
            o_f64[bi * d + j] = o[j];
            lo = std::fmin(lo, o[j]);
            hi = std::fmax(hi, o[j]);
        }
        uint16_t lo16 = orc_double_to_half(lo), st16 = orc_double_to_half((hi - lo) / 15.0);
        if (in_o) {
            lo16 = (uint16_t)(side_in[bi * R] | (side_in[bi * R + 1] << 8));
            st16 = (uint16_t)(side_in[bi * R + 2] | (side_in[bi * R + 3] << 8));
        }
        const double lov = orc_half_to_double(lo16), stv = orc_half_to_double(st16);
        rec[0] = (uint8_t)(lo16 & 0xFF);
        rec[1] = (uint8_t)(lo16 >> 8);
        rec[2] = (uint8_t)(st16 & 0xFF);
        rec[3] = (uint8_t)(st16 >> 8);
        for (int j = 0; j < d; ++j) {
            int q;
            if (in_o) {
                const uint8_t by = side_in[bi * R + 8 + j / 2];
                q = (j & 1) ? (by >> 4) : (by & 15);
            } else if (stv == 0.0) {
                q = 0;
            } else {
                q = (int)std::nearbyint((o[j] - lov) / stv);
                q = q < 0 ? 0 : (q > 15 ? 15 : q);
            }
            rec[8 + j / 2] |= (uint8_t)(q << ((j & 1) * 4));
            o_hat[bi * d + j] = (double)(float)(lov + stv * q);
        }
        // the shifted tokens, coded without QJL
        for (int t = 0; t < blk; ++t) {
            for (int j = 0; j < d; ++j) w[j] = u[(size_t)t * d + j] - o_hat[bi * d + j];
            double nw = 0.0, gam = 0.0;
            orc_quantize(d, b, 0, 0, delta, nullptr, centroid, threshold, w.data(), 1, codes + (b0 + t) * d, nullptr,
                         &nw, &gam, z_out ? z_out + (b0 + t) * d : nullptr, nullptr);
            norm_w[b0 + t] = nw;
        }
    }
}

}  // extern "C"
