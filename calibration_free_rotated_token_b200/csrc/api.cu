// api.cu -- the C ABI of include/kvq.h: argument checks, the per-handle
// constants (signs, Gaussian projection, Lloyd-Max codebook), TMA tensor
// maps and kernel dispatch.  Host code only.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/kvq.h"
#include "kvq_internal.h"

namespace kvq {
// One per (d, b), from quantize_inst.cu.
cudaError_t launch_quantize_d64_b1(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d64_b2(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d64_b3(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d64_b4(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d128_b1(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d128_b2(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d128_b3(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d128_b4(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d256_b1(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d256_b2(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d256_b3(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);
cudaError_t launch_quantize_d256_b4(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                  int dtype, const QuantArgs& a, int sms, cudaStream_t s);

namespace {
cudaError_t launch_quantize_any(int d, int b, bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                int dtype, const QuantArgs& a, int sms, cudaStream_t s) {
#define KVQ_CASE(D, B) \
    if (d == D && b == B) return launch_quantize_d##D##_b##B(qjl, nsn, map, map1, dtype, a, sms, s);
    KVQ_CASE(64, 1) KVQ_CASE(64, 2) KVQ_CASE(64, 3) KVQ_CASE(64, 4)
    KVQ_CASE(128, 1) KVQ_CASE(128, 2) KVQ_CASE(128, 3) KVQ_CASE(128, 4)
    KVQ_CASE(256, 1) KVQ_CASE(256, 2) KVQ_CASE(256, 3) KVQ_CASE(256, 4)
#undef KVQ_CASE
    return cudaErrorNotSupported;
}
}  // namespace
}  // namespace kvq

static_assert(kvq::kMaxWindow == KVQ_MAX_WINDOW, "window bound of the header and the kernels");

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
    g_err = msg;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(KVQ_ECUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

// ---------------------------------------------------------------------------
// Constants of a handle.  The pages draw random signs and a Gaussian
// projection without naming a generator; this library uses SplitMix64
// (Steele, Lea, Flood, OOPSLA 2014): output i of the stream seeded with s is
// the finaliser applied to s + (i + 1) * 0x9E3779B97F4A7C15.
// ---------------------------------------------------------------------------
uint64_t sm64(uint64_t seed, uint64_t i) {
    uint64_t x = seed + (i + 1) * 0x9E3779B97F4A7C15ULL;
    x ^= x >> 30;
    x *= 0xBF58476D1CE4E5B9ULL;
    x ^= x >> 27;
    x *= 0x94D049BB133111EBULL;
    x ^= x >> 31;
    return x;
}

// Normal draw number k of stream `seed`: Box-Muller (cosine branch) on the
// top 53 bits of outputs 2k (shifted into (0, 1]) and 2k+1 (in [0, 1)).
double normal_draw(uint64_t seed, uint64_t k) {
    const double two53 = 9007199254740992.0;
    const double u1 = static_cast<double>((sm64(seed, 2 * k) >> 11) + 1) / two53;
    const double u2 = static_cast<double>(sm64(seed, 2 * k + 1) >> 11) / two53;
    return std::sqrt(-2.0 * std::log(u1)) * std::cos(6.283185307179586476925286766559 * u2);
}

double phi(double x) { return std::isinf(x) ? 0.0 : 0.39894228040143267794 * std::exp(-0.5 * x * x); }
double Phi(double x) {
    if (std::isinf(x)) return x > 0 ? 1.0 : 0.0;
    return 0.5 * std::erfc(-0.70710678118654752440 * x);
}

// Gaussian Lloyd-Max codebook with L = 2^b levels (PolarQuant section 2:
// Lloyd-Max centroids for N(0, 1); TurboQuant "Como Implementar": codebooks
// precomputed per bit width).  Fixed-point iteration on the interior
// decision levels: given decision levels, each centroid is the conditional
// mean of its cell; the new decision levels are the centroid midpoints.
void lloyd_max_codebook(int b, std::vector<double>* cent, std::vector<double>* thr) {
    const int L = 1 << b;
    std::vector<double> t(L + 1), c(L);
    for (int k = 0; k <= L; ++k) t[k] = (k == 0) ? -INFINITY : (k == L ? INFINITY : -3.0 + 6.0 * k / L);
    for (int iter = 0; iter < 1000000; ++iter) {
        for (int k = 0; k < L; ++k) c[k] = (phi(t[k]) - phi(t[k + 1])) / (Phi(t[k + 1]) - Phi(t[k]));
        double change = 0.0;
        for (int k = 1; k < L; ++k) {
            const double nt = 0.5 * (c[k - 1] + c[k]);
            change = std::fmax(change, std::fabs(nt - t[k]));
            t[k] = nt;
        }
        if (change <= 1e-15) break;
    }
    for (int k = 0; k < L; ++k) c[k] = (phi(t[k]) - phi(t[k + 1])) / (Phi(t[k + 1]) - Phi(t[k]));
    // N(0, 1) is symmetric, so is its optimal codebook: remove the rounding
    // asymmetry, which also makes the middle decision level exactly 0.
    for (int k = 0; k < L / 2; ++k) {
        const double m = 0.5 * (c[L - 1 - k] - c[k]);
        c[k] = -m;
        c[L - 1 - k] = m;
    }
    cent->assign(c.begin(), c.end());
    thr->clear();
    for (int k = 1; k < L; ++k) thr->push_back(0.5 * (c[k - 1] + c[k]));
}

// Codebook for the exact law of one coordinate of a rotated unit vector,
// scaled by sqrt(d) (TurboQuant blog, "Estágio 1": Beta((d-1)/2, (d-1)/2) on
// [-1, 1], Lloyd-Max over it).  Density of z: f(z) ~ (1 - z^2/d)^a on
// |z| < sqrt(d), a = (d-3)/2.  Cell moments in closed form:
//   int_0^t f  ~ sqrt(d) I_n(asin(t/sqrt(d))),  I_n(th) = int_0^th cos^n,
//                n = d - 2, by I_n = cos^(n-1) sin / n + (n-1)/n I_(n-2);
//   int z f    ~ -d/(d-1) (1 - t^2/d)^((d-1)/2)  (antiderivative).
// The common normalisation cancels in every centroid (a ratio of the two).
double sphere_m0(int d, double t) {
    const double r = std::sqrt(static_cast<double>(d));
    const double x = std::fmin(std::fabs(t) / r, 1.0);
    const double th = std::asin(x), sn = std::sin(th), cs = std::cos(th);
    const int n = d - 2;
    double I = (n % 2 == 0) ? th : sn;  // I_0 or I_1
    double cp = (n % 2 == 0) ? cs : cs * cs;  // cos^(k-1) for the first step k = 2 or 3
    for (int k = (n % 2 == 0) ? 2 : 3; k <= n; k += 2) {
        I = cp * sn / k + (k - 1.0) / k * I;
        cp *= cs * cs;
    }
    return std::copysign(r * I, t);
}
double sphere_f1(int d, double t) {
    const double w = std::fmax(1.0 - t * t / d, 0.0);
    return -static_cast<double>(d) / (d - 1) * std::pow(w, 0.5 * (d - 1));
}

void lloyd_max_sphere_codebook(int d, int b, std::vector<double>* cent, std::vector<double>* thr) {
    const int L = 1 << b;
    const double edge = std::sqrt(static_cast<double>(d));
    std::vector<double> c, t0;
    lloyd_max_codebook(b, &c, &t0);  // starting point: the Gaussian codebook, inside the support
    double mx = 0.0;
    for (double v : c) mx = std::fmax(mx, std::fabs(v));
    if (mx > 0.9 * edge)
        for (double& v : c) v *= 0.9 * edge / mx;
    std::vector<double> t(L + 1);
    for (int iter = 0; iter < 1000000; ++iter) {
        t[0] = -edge;
        t[L] = edge;
        for (int k = 1; k < L; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
        double change = 0.0;
        for (int k = 0; k < L; ++k) {
            const double m0 = sphere_m0(d, t[k + 1]) - sphere_m0(d, t[k]);
            const double nc = (sphere_f1(d, t[k + 1]) - sphere_f1(d, t[k])) / m0;
            change = std::fmax(change, std::fabs(nc - c[k]));
            c[k] = nc;
        }
        if (change <= 1e-15) break;
    }
    for (int k = 0; k < L / 2; ++k) {
        const double m = 0.5 * (c[L - 1 - k] - c[k]);
        c[k] = -m;
        c[L - 1 - k] = m;
    }
    cent->assign(c.begin(), c.end());
    thr->clear();
    for (int k = 1; k < L; ++k) thr->push_back(0.5 * (c[k - 1] + c[k]));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over rows x d elements (row stride ld elements), box 128 bytes x
// 128 rows, 128-byte swizzle, zero fill out of bounds.
int make_row_map(CUtensorMap* map, const void* x, int dtype, int64_t rows, int d, int64_t ld) {
    auto enc = encode_fn();
    if (!enc) return fail(KVQ_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int esz = dtype == KVQ_F32 ? 4 : 2;
    const CUtensorMapDataType dt = dtype == KVQ_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dtype == KVQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t gstride[1] = {static_cast<cuuint64_t>(ld) * esz};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 128u};
    cuuint32_t estride[2] = {1u, 1u};
    CUresult r = enc(map, dt, 2, const_cast<void*>(x), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KVQ_ECUDA, "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(r));
    return KVQ_OK;
}

int check_handle(const kvq_ctx* h) {
    if (!h) return fail(KVQ_EINVAL, "null handle");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != h->device)
        return fail(KVQ_EINVAL, "handle was created on device " + std::to_string(h->device) +
                                    " but the current device is " + std::to_string(dev));
    return KVQ_OK;
}

void fill_common(const kvq_ctx* h, float* cent, float* thr, uint32_t* ps) {
    for (int k = 0; k < kvq::kMaxLevels; ++k) {
        cent[k] = k < static_cast<int>(h->centroids.size()) ? h->centroids[k] : 0.f;
        thr[k] = k < static_cast<int>(h->thresholds.size()) ? h->thresholds[k] : INFINITY;
    }
    std::memcpy(ps, h->pair_sign, sizeof(h->pair_sign));
}

// One stream of vectors to quantize.
struct QJob {
    const void* x;
    int dtype;
    int64_t rows, ld;
    int layout;
    uint32_t* codes;
    uint32_t* qjl;
    uint16_t* norms;
};

// Argument checks of one stream; builds its tensor map when rows > 0.
int check_job(kvq_handle h, const QJob& j, bool nsn, CUtensorMap* map) {
    if (j.dtype != KVQ_F32 && j.dtype != KVQ_F16 && j.dtype != KVQ_BF16) return fail(KVQ_EINVAL, "unknown dtype");
    if (j.layout != KVQ_LAYOUT_TOKEN && j.layout != KVQ_LAYOUT_BLOCK32) return fail(KVQ_EINVAL, "unknown layout");
    if (j.rows < 0) return fail(KVQ_EINVAL, "negative vector count");
    if (j.rows == 0) return KVQ_OK;
    if (j.rows > (int64_t(1) << 31) - 128) return fail(KVQ_EINVAL, "more than 2^31 - 128 vectors in one call");
    const int esz = j.dtype == KVQ_F32 ? 4 : 2;
    if (j.ld < h->d) return fail(KVQ_EINVAL, "row stride ld is smaller than d");
    if ((j.ld * esz) % 16 != 0) return fail(KVQ_EINVAL, "row stride ld * element size must be a multiple of 16 bytes");
    if (!j.x || !aligned(j.x, 16)) return fail(KVQ_EINVAL, "x must be a non-null 16-byte aligned device pointer");
    if (!j.codes || !aligned(j.codes, 16)) return fail(KVQ_EINVAL, "codes must be non-null and 16-byte aligned");
    if (!j.norms || !aligned(j.norms, 4)) return fail(KVQ_EINVAL, "norms must be non-null and 4-byte aligned");
    const bool has_qjl = (h->flags & KVQ_QJL) != 0;
    if (!nsn) {
        if (has_qjl && (!j.qjl || !aligned(j.qjl, 16)))
            return fail(KVQ_EINVAL, "qjl must be non-null and 16-byte aligned");
        if (!has_qjl && j.qjl) return fail(KVQ_EINVAL, "qjl must be NULL for a handle without KVQ_QJL");
    }
    if (j.dtype == KVQ_F32 && h->d > 128) return fail(KVQ_EUNSUPPORTED, "fp32 input is built for d <= 128");
    return make_row_map(map, j.x, j.dtype, j.rows, h->d, j.ld);
}

// One launch over one stream (j1 == nullptr) or two streams of the same
// dtype (the tensor-core kernel's tiles of j0, then those of j1).
int launch_jobs(kvq_handle h, const QJob& j0, const CUtensorMap& m0, const QJob* j1, const CUtensorMap* m1,
                uint16_t* block_mean, bool nsn, void* stream, uint8_t* side = nullptr) {
    kvq::QuantArgs a{};
    a.n = j0.rows;
    a.layout = j0.layout;
    a.ntiles0 = (j0.rows + kvq::kTileRows - 1) / kvq::kTileRows;
    a.ntiles = a.ntiles0;
    a.codes = j0.codes;
    a.qjl = nsn ? nullptr : j0.qjl;
    a.norms = reinterpret_cast<__half2*>(j0.norms);
    if (j1) {
        a.n1 = j1->rows;
        a.layout1 = j1->layout;
        a.ntiles += (j1->rows + kvq::kTileRows - 1) / kvq::kTileRows;
        a.codes1 = j1->codes;
        a.qjl1 = j1->qjl;
        a.norms1 = reinterpret_cast<__half2*>(j1->norms);
    }
    a.block_mean = reinterpret_cast<__half*>(block_mean);
    a.side = side;
    a.cuda_core_rotation = (h->flags & KVQ_CUDA_CORE_ROTATION) != 0 && !nsn;
    a.S = h->d_S;
    a.status = h->d_status;
    fill_common(h, a.centroid, a.threshold, a.pair_sign);
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool has_qjl = (h->flags & KVQ_QJL) != 0;
    const cudaError_t err =
        kvq::launch_quantize_any(h->d, h->b, has_qjl, nsn, m0, j1 ? *m1 : m0, j0.dtype, a, sms, s);
    if (err == cudaErrorNotSupported) return fail(KVQ_EUNSUPPORTED, "this (d, dtype, front end) is not built");
    if (err != cudaSuccess) return cuda_fail(err, "quantize launch");
    return KVQ_OK;
}

int quantize_common(kvq_handle h, const void* x, int dtype, int64_t rows, int64_t ld, int layout, uint32_t* codes,
                    uint32_t* qjl, uint16_t* norms, uint16_t* block_mean, bool nsn, void* stream,
                    uint8_t* side = nullptr) {
    if (int e = check_handle(h)) return e;
    const QJob j{x, dtype, rows, ld, layout, codes, qjl, norms};
    CUtensorMap map;
    if (int e = check_job(h, j, nsn, &map)) return e;
    if (rows == 0) return KVQ_OK;
    return launch_jobs(h, j, map, nullptr, nullptr, block_mean, nsn, stream, side);
}

// Bytes of one side record of the double-quantized NSN front end (d = 64, 128).
size_t dq_side_bytes(int d) { return static_cast<size_t>((8 + d / 2 + 64 + 15) / 16 * 16); }

}  // namespace

extern "C" {

const char* kvq_last_error(void) { return g_err.c_str(); }

int kvq_init(kvq_handle* out, int d, int b, uint64_t seed, uint32_t flags) {
    g_err.clear();
    if (!out) return fail(KVQ_EINVAL, "null output handle pointer");
    *out = nullptr;
    if (d != 64 && d != 128 && d != 256) return fail(KVQ_EINVAL, "d must be 64, 128 or 256");
    if (b < 1 || b > 4) return fail(KVQ_EINVAL, "b must be in 1..4");
    if (flags & ~(KVQ_QJL | KVQ_BETA_CODEBOOK | KVQ_CUDA_CORE_ROTATION)) return fail(KVQ_EINVAL, "unknown flag bits");
    kvq_ctx* h = new (std::nothrow) kvq_ctx();
    if (!h) return fail(KVQ_ENOMEM, "host allocation failed");
    cudaGetDevice(&h->device);
    h->d = d;
    h->b = b;
    h->m = d;
    h->flags = flags;
    h->seed = seed;
    h->signs.resize(d);
    for (int j = 0; j < d; ++j) h->signs[j] = (sm64(seed, static_cast<uint64_t>(j)) >> 63) ? -1 : 1;
    for (int k = 0; k < d / 2; ++k)
        h->pair_sign[k] = (h->signs[2 * k] < 0 ? 0x8000u : 0u) | (h->signs[2 * k + 1] < 0 ? 0x80000000u : 0u);
    h->S_half.resize(static_cast<size_t>(h->m) * d);
    for (size_t k = 0; k < h->S_half.size(); ++k) {
        const __half v = __double2half(normal_draw(seed + 1, k));
        std::memcpy(&h->S_half[k], &v, 2);
    }
    std::vector<double> c, t;
    if (flags & KVQ_BETA_CODEBOOK) lloyd_max_sphere_codebook(d, b, &c, &t);
    else lloyd_max_codebook(b, &c, &t);
    h->centroids.assign(c.begin(), c.end());
    h->thresholds.assign(t.begin(), t.end());
    cudaError_t e = cudaMalloc(&h->d_S, h->S_half.size() * sizeof(__half));
    if (e == cudaSuccess) e = cudaMalloc(&h->d_status, sizeof(uint32_t));
    if (e == cudaSuccess)
        e = cudaMemcpy(h->d_S, h->S_half.data(), h->S_half.size() * sizeof(__half), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(h->d_status, 0, sizeof(uint32_t));
    if (e != cudaSuccess) {
        cudaFree(h->d_S);
        cudaFree(h->d_status);
        delete h;
        return e == cudaErrorMemoryAllocation ? fail(KVQ_ENOMEM, "device allocation failed")
                                              : cuda_fail(e, "kvq_init");
    }
    *out = h;
    return KVQ_OK;
}

int kvq_codebook(int d, int b, uint32_t flags, float* centroids, float* thresholds) {
    g_err.clear();
    if (d != 64 && d != 128 && d != 256) return fail(KVQ_EINVAL, "d must be 64, 128 or 256");
    if (b < 1 || b > 4) return fail(KVQ_EINVAL, "b must be in 1..4");
    if (flags & ~(KVQ_QJL | KVQ_BETA_CODEBOOK | KVQ_CUDA_CORE_ROTATION)) return fail(KVQ_EINVAL, "unknown flag bits");
    if (!centroids || !thresholds) return fail(KVQ_EINVAL, "centroids and thresholds must be non-null");
    std::vector<double> c, t;
    if (flags & KVQ_BETA_CODEBOOK) lloyd_max_sphere_codebook(d, b, &c, &t);
    else lloyd_max_codebook(b, &c, &t);
    for (size_t k = 0; k < c.size(); ++k) centroids[k] = static_cast<float>(c[k]);
    for (size_t k = 0; k < t.size(); ++k) thresholds[k] = static_cast<float>(t[k]);
    return KVQ_OK;
}

int kvq_destroy(kvq_handle h) {
    g_err.clear();
    if (!h) return KVQ_OK;
    cudaFree(h->d_S);
    cudaFree(h->d_status);
    delete h;
    return KVQ_OK;
}

int kvq_get_info(kvq_handle h, int* d, int* b, int* m, uint32_t* flags) {
    g_err.clear();
    if (!h) return fail(KVQ_EINVAL, "null handle");
    if (d) *d = h->d;
    if (b) *b = h->b;
    if (m) *m = h->m;
    if (flags) *flags = h->flags;
    return KVQ_OK;
}

int kvq_get_constants(kvq_handle h, int8_t* signs, uint16_t* S, float* centroids, float* thresholds) {
    g_err.clear();
    if (!h) return fail(KVQ_EINVAL, "null handle");
    if (signs) std::memcpy(signs, h->signs.data(), h->signs.size());
    if (S) std::memcpy(S, h->S_half.data(), h->S_half.size() * 2);
    if (centroids) std::memcpy(centroids, h->centroids.data(), h->centroids.size() * sizeof(float));
    if (thresholds) std::memcpy(thresholds, h->thresholds.data(), h->thresholds.size() * sizeof(float));
    return KVQ_OK;
}

int kvq_quantize(kvq_handle h, const void* x, int dtype, int64_t n, int64_t ld, int layout, uint32_t* codes,
                 uint32_t* qjl, uint16_t* norms, void* stream) {
    g_err.clear();
    return quantize_common(h, x, dtype, n, ld, layout, codes, qjl, norms, nullptr, false, stream);
}

int kvq_quantize_batch(kvq_handle h, int count, const kvq_quant_job* jobs, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (count < 0 || (count > 0 && !jobs)) return fail(KVQ_EINVAL, "count must be >= 0 and jobs non-null");
    std::vector<QJob> js;
    std::vector<CUtensorMap> maps;
    js.reserve(count);
    maps.reserve(count);
    for (int i = 0; i < count; ++i) {
        const kvq_quant_job& u = jobs[i];
        const QJob j{u.x, u.dtype, u.n, u.ld, u.layout, u.codes, u.qjl, u.norms};
        CUtensorMap m;
        if (int e = check_job(h, j, false, &m)) return fail(e, "job " + std::to_string(i) + ": " + g_err);
        if (j.rows == 0) continue;
        js.push_back(j);
        maps.push_back(m);
    }
    for (size_t i = 0; i < js.size();) {
        const bool pair = i + 1 < js.size() && js[i].dtype == js[i + 1].dtype &&
                          kvq::quantize_pairs(h->d, js[i].dtype, false, (h->flags & KVQ_QJL) != 0) &&
                          !(h->flags & KVQ_CUDA_CORE_ROTATION);
        if (int e = launch_jobs(h, js[i], maps[i], pair ? &js[i + 1] : nullptr, pair ? &maps[i + 1] : nullptr,
                                nullptr, false, stream))
            return e;
        i += pair ? 2 : 1;
    }
    return KVQ_OK;
}

int kvq_nsn_quantize(kvq_handle h, const void* x, int dtype, int64_t n_heads, int64_t n_tok, int layout,
                     uint32_t* codes, uint16_t* norms, uint16_t* block_mean, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "the NSN front end takes a handle without KVQ_QJL");
    if (n_heads < 0 || n_tok < 0) return fail(KVQ_EINVAL, "negative size");
    if (n_tok % 128 != 0) return fail(KVQ_EINVAL, "n_tok must be a multiple of 128 (NSN blocks of 128 tokens)");
    if (h->d > 128 && dtype == KVQ_F32)
        return fail(KVQ_EUNSUPPORTED, "the NSN front end at d = 256 is built for fp16 and bf16 input");
    if (n_heads * n_tok == 0) return KVQ_OK;
    if (!block_mean || !aligned(block_mean, 2)) return fail(KVQ_EINVAL, "block_mean must be non-null");
    return quantize_common(h, x, dtype, n_heads * n_tok, h->d, layout, codes, nullptr, norms, block_mean, true,
                           stream);
}

size_t kvq_nsn_dq_side_bytes(int d) { return (d == 64 || d == 128 || d == 256) ? dq_side_bytes(d) : 0; }

int kvq_nsn_dq_quantize(kvq_handle h, const void* x, int dtype, int64_t n_heads, int64_t n_tok, int layout,
                        uint32_t* codes, uint16_t* wnorms, uint8_t* side, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "the NSN front end takes a handle without KVQ_QJL");
    if (n_heads < 0 || n_tok < 0) return fail(KVQ_EINVAL, "negative size");
    if (n_tok % 128 != 0) return fail(KVQ_EINVAL, "n_tok must be a multiple of 128 (NSN blocks of 128 tokens)");
    if (dtype != KVQ_F16 && dtype != KVQ_BF16)
        return fail(dtype == KVQ_F32 ? KVQ_EUNSUPPORTED : KVQ_EINVAL,
                    "double-quantized NSN side data are built for fp16 and bf16 input");
    if (n_heads * n_tok == 0) return KVQ_OK;
    if (!side || !aligned(side, 16)) return fail(KVQ_EINVAL, "side must be non-null and 16-byte aligned");
    return quantize_common(h, x, dtype, n_heads * n_tok, h->d, layout, codes, nullptr, wnorms, nullptr, true,
                           stream, side);
}

size_t kvq_decode_workspace(kvq_handle h, int batch, int hq, int hkv, int64_t max_T) {
    if (!h || batch <= 0 || hq <= 0 || hkv <= 0 || max_T < 0) return 0;
    int ns = 0;
    int64_t chunk = 0;
    size_t ws = 0;
    kvq::decode_plan(h, batch, hq, hkv, max_T > 0 ? max_T : 1, &ns, &chunk, &ws);
    return ws;
}

}  // extern "C"

namespace {

// Argument checks shared by both decode entry points; fills the split plan.
int decode_check(kvq_handle h, int dtype, int batch, int hq, int hkv, const kvq_cache* k, const kvq_cache* v,
                 const void* q, const int32_t* seq_len, int64_t max_T, float scale, float* out, int* ns,
                 int64_t* chunk, size_t* need) {
    if (int e = check_handle(h)) return e;
    if (dtype != KVQ_F32 && dtype != KVQ_F16 && dtype != KVQ_BF16) return fail(KVQ_EINVAL, "unknown dtype");
    if (batch <= 0 || hq <= 0 || hkv <= 0) return fail(KVQ_EINVAL, "batch, hq and hkv must be positive");
    if (hq % hkv != 0) return fail(KVQ_EINVAL, "hq must be a multiple of hkv");
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return fail(KVQ_EUNSUPPORTED, "hq / hkv must be 1, 2, 4 or 8");
    if (max_T < 0) return fail(KVQ_EINVAL, "negative max_T");
    if (!k || !v) return fail(KVQ_EINVAL, "null cache descriptor");
    const bool has_qjl = (h->flags & KVQ_QJL) != 0;
    for (const kvq_cache* c : {k, v}) {
        if (!c->codes || !aligned(c->codes, 4) || !c->norms || !aligned(c->norms, 4))
            return fail(KVQ_EINVAL, "cache codes/norms must be non-null and 4-byte aligned");
        if (has_qjl && (!c->qjl || !aligned(c->qjl, 4))) return fail(KVQ_EINVAL, "cache qjl must be non-null");
        if (c->capacity < max_T) return fail(KVQ_EINVAL, "cache capacity is smaller than max_T");
    }
    if (k->layout != KVQ_LAYOUT_TOKEN) return fail(KVQ_EINVAL, "the key cache must use KVQ_LAYOUT_TOKEN");
    if (v->layout != KVQ_LAYOUT_BLOCK32) return fail(KVQ_EINVAL, "the value cache must use KVQ_LAYOUT_BLOCK32");
    if (k->capacity % 32 != 0 || v->capacity % 32 != 0)
        return fail(KVQ_EINVAL, "cache capacities must be multiples of 32");
    for (const kvq_cache* c : {k, v}) {
        if (!aligned(c->codes, 16) || !aligned(c->norms, 16) || (c->qjl && !aligned(c->qjl, 16)))
            return fail(KVQ_EINVAL, "cache buffers must be 16-byte aligned");
    }
    if (!q || !out || !seq_len) return fail(KVQ_EINVAL, "q, out and seq_len must be non-null");
    if (!std::isfinite(scale)) return fail(KVQ_EINVAL, "scale must be finite");
    kvq::decode_plan(h, batch, hq, hkv, max_T > 0 ? max_T : 1, ns, chunk, need);
    return KVQ_OK;
}

// Optional parts of a decode call: NSN block means, a residual window, the
// logits row stride.
struct DecodeExtras {
    bool dq = false;  // kmean / vmean are double-quantized side records; norms hold fp16 ||w||
    const uint16_t* kmean = nullptr;
    const uint16_t* vmean = nullptr;
    const uint16_t* kwin = nullptr;
    const uint16_t* vwin = nullptr;
    int64_t win_cap = 0;
    const int32_t* win_len = nullptr;
    int64_t logits_ld = 0;
};

int decode_launch(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                  const kvq_cache* v, const int32_t* seq_len, int64_t max_T, float scale, float* logits,
                  float* out, void* workspace, int ns, int64_t chunk, void* stream,
                  const DecodeExtras& x = DecodeExtras()) {
    kvq::DecodeArgs a{};
    a.nsn = x.kmean != nullptr;
    a.nsn_dq = x.dq ? 1 : 0;
    a.kmean = reinterpret_cast<const __half*>(x.kmean);
    a.vmean = reinterpret_cast<const __half*>(x.vmean);
    a.kwin = reinterpret_cast<const __half*>(x.kwin);
    a.vwin = reinterpret_cast<const __half*>(x.vwin);
    a.win_cap = x.win_cap;
    a.win_len = x.win_len;
    a.win_dim = h->d;
    a.logits_ld = x.logits_ld > 0 ? x.logits_ld : max_T;
    a.batch = batch;
    a.hq = hq;
    a.hkv = hkv;
    a.G = hq / hkv;
    a.max_T = max_T;
    a.nsplit_run = ns;
    a.nsplit = ns + (x.kwin != nullptr ? 1 : 0);  // the window's partial is the last split
    a.chunk = chunk;
    a.q = q;
    a.qdtype = dtype;
    a.kcodes = k->codes;
    a.kqjl = k->qjl;
    a.knorms = reinterpret_cast<const __half2*>(k->norms);
    a.vcodes = v->codes;
    a.vqjl = v->qjl;
    a.vnorms = reinterpret_cast<const __half2*>(v->norms);
    a.kcap = k->capacity;
    a.vcap = v->capacity;
    a.seq_len = seq_len;
    a.scale = scale;
    a.logits = logits;
    a.out = out;
    const int64_t bh = static_cast<int64_t>(batch) * hq;
    const int64_t streams = static_cast<int64_t>(batch) * hkv;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    size_t off = static_cast<size_t>(bh * (ns + 1) * (2 + h->d + h->m)) * sizeof(float);
    off = (off + 255) / 256 * 256;
    a.part = reinterpret_cast<float*>(ws);
    if (kvq::decode_uses_mma(h)) {
        a.qscal = reinterpret_cast<float*>(ws + off);
        off += static_cast<size_t>(bh) * 4 * sizeof(float);
        off = (off + 255) / 256 * 256;
        a.qfrag = reinterpret_cast<uint2*>(ws + off);
        (void)streams;
    } else {
        a.qrot = reinterpret_cast<float*>(ws + off);
        a.qproj = a.qrot + bh * h->d;
    }
    a.S = h->d_S;
    a.status = h->d_status;
    float thr_unused[kvq::kMaxLevels];
    fill_common(h, a.centroid, thr_unused, a.pair_sign);
    std::string why;
    cudaError_t e = kvq::launch_decode(h, a, static_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess) return cuda_fail(e, ("decode launch " + why).c_str());
    return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                      const kvq_cache* v, const int32_t* seq_len, int64_t max_T, float scale, float* logits,
                      float* out, void* workspace, size_t ws_bytes, void* stream) {
    g_err.clear();
    int ns = 0;
    int64_t chunk = 0;
    size_t need = 0;
    if (int e = decode_check(h, dtype, batch, hq, hkv, k, v, q, seq_len, max_T, scale, out, &ns, &chunk, &need))
        return e;
    if (!workspace || !aligned(workspace, 16)) return fail(KVQ_EINVAL, "workspace must be non-null and 16-byte aligned");
    if (ws_bytes < need) return fail(KVQ_EINVAL, "workspace too small: need " + std::to_string(need) + " bytes");
    return decode_launch(h, q, dtype, batch, hq, hkv, k, v, seq_len, max_T, scale, logits, out, workspace, ns, chunk,
                         stream);
}

int kvq_nsn_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                          const kvq_cache* v, const uint16_t* k_block_mean, const uint16_t* v_block_mean,
                          const int32_t* seq_len, int64_t max_T, float scale, float* logits, float* out,
                          void* workspace, size_t ws_bytes, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "NSN caches carry no QJL sketch: use a handle without KVQ_QJL");
    int ns = 0;
    int64_t chunk = 0;
    size_t need = 0;
    if (int e = decode_check(h, dtype, batch, hq, hkv, k, v, q, seq_len, max_T, scale, out, &ns, &chunk, &need))
        return e;
    if (k->capacity % 128 != 0 || v->capacity % 128 != 0)
        return fail(KVQ_EINVAL, "NSN cache capacities must be multiples of 128 (one block mean per 128 tokens)");
    if (!k_block_mean || !v_block_mean || !aligned(k_block_mean, 16) || !aligned(v_block_mean, 16))
        return fail(KVQ_EINVAL, "block means must be non-null and 16-byte aligned");
    if (!workspace || !aligned(workspace, 16)) return fail(KVQ_EINVAL, "workspace must be non-null and 16-byte aligned");
    if (ws_bytes < need) return fail(KVQ_EINVAL, "workspace too small: need " + std::to_string(need) + " bytes");
    DecodeExtras x;
    x.kmean = k_block_mean;
    x.vmean = v_block_mean;
    return decode_launch(h, q, dtype, batch, hq, hkv, k, v, seq_len, max_T, scale, logits, out, workspace, ns, chunk,
                         stream, x);
}

int kvq_nsn_dq_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                             const kvq_cache* v, const uint8_t* k_side, const uint8_t* v_side, const int32_t* seq_len,
                             int64_t max_T, float scale, float* logits, float* out, void* workspace, size_t ws_bytes,
                             void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "NSN caches carry no QJL sketch: use a handle without KVQ_QJL");
    int ns = 0;
    int64_t chunk = 0;
    size_t need = 0;
    if (int e = decode_check(h, dtype, batch, hq, hkv, k, v, q, seq_len, max_T, scale, out, &ns, &chunk, &need))
        return e;
    if (k->capacity % 128 != 0 || v->capacity % 128 != 0)
        return fail(KVQ_EINVAL, "NSN cache capacities must be multiples of 128 (one side record per 128 tokens)");
    if (!k_side || !v_side || !aligned(k_side, 16) || !aligned(v_side, 16))
        return fail(KVQ_EINVAL, "side records must be non-null and 16-byte aligned");
    if (!workspace || !aligned(workspace, 16)) return fail(KVQ_EINVAL, "workspace must be non-null and 16-byte aligned");
    if (ws_bytes < need) return fail(KVQ_EINVAL, "workspace too small: need " + std::to_string(need) + " bytes");
    DecodeExtras x;
    x.dq = true;
    x.kmean = reinterpret_cast<const uint16_t*>(k_side);
    x.vmean = reinterpret_cast<const uint16_t*>(v_side);
    return decode_launch(h, q, dtype, batch, hq, hkv, k, v, seq_len, max_T, scale, logits, out, workspace, ns, chunk,
                         stream, x);
}

int kvq_decode_attend_ex(kvq_handle h, const kvq_decode_desc* d, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (!d) return fail(KVQ_EINVAL, "null descriptor");
    int ns = 0;
    int64_t chunk = 0;
    size_t need = 0;
    if (int e = decode_check(h, d->dtype, d->batch, d->hq, d->hkv, d->k, d->v, d->q, d->seq_len, d->max_T, d->scale,
                             d->out, &ns, &chunk, &need))
        return e;
    DecodeExtras x;
    if (d->k_side || d->v_side) {
        if (d->k_block_mean || d->v_block_mean)
            return fail(KVQ_EINVAL, "side records and block means describe different caches: give one kind");
        if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "NSN caches carry no QJL sketch: use a handle without KVQ_QJL");
        if (!d->k_side || !d->v_side || !aligned(d->k_side, 16) || !aligned(d->v_side, 16))
            return fail(KVQ_EINVAL, "side records must both be non-null and 16-byte aligned");
        if (d->k->capacity % 128 != 0 || d->v->capacity % 128 != 0)
            return fail(KVQ_EINVAL, "NSN cache capacities must be multiples of 128 (one side record per 128 tokens)");
        x.dq = true;
        x.kmean = reinterpret_cast<const uint16_t*>(d->k_side);
        x.vmean = reinterpret_cast<const uint16_t*>(d->v_side);
    }
    if (d->k_block_mean || d->v_block_mean) {
        if (h->flags & KVQ_QJL) return fail(KVQ_EINVAL, "NSN caches carry no QJL sketch: use a handle without KVQ_QJL");
        if (!d->k_block_mean || !d->v_block_mean || !aligned(d->k_block_mean, 16) || !aligned(d->v_block_mean, 16))
            return fail(KVQ_EINVAL, "block means must both be non-null and 16-byte aligned");
        if (d->k->capacity % 128 != 0 || d->v->capacity % 128 != 0)
            return fail(KVQ_EINVAL, "NSN cache capacities must be multiples of 128 (one block mean per 128 tokens)");
        x.kmean = d->k_block_mean;
        x.vmean = d->v_block_mean;
    }
    if (d->k_window || d->v_window) {
        if (!d->k_window || !d->v_window || !d->window_len || !aligned(d->k_window, 16) || !aligned(d->v_window, 16))
            return fail(KVQ_EINVAL, "the window needs k_window, v_window (16-byte aligned) and window_len");
        if (d->window_cap < 1 || d->window_cap > KVQ_MAX_WINDOW)
            return fail(KVQ_EINVAL, "window_cap must be in 1.." + std::to_string(KVQ_MAX_WINDOW));
        x.kwin = d->k_window;
        x.vwin = d->v_window;
        x.win_cap = d->window_cap;
        x.win_len = d->window_len;
    }
    const int64_t row = d->max_T + (x.kwin ? d->window_cap : 0);
    if (d->logits && d->logits_ld != 0 && d->logits_ld < row)
        return fail(KVQ_EINVAL, "logits_ld must be at least max_T (+ window_cap with a window)");
    x.logits_ld = d->logits_ld != 0 ? d->logits_ld : row;
    if (!d->workspace || !aligned(d->workspace, 16))
        return fail(KVQ_EINVAL, "workspace must be non-null and 16-byte aligned");
    if (d->ws_bytes < need) return fail(KVQ_EINVAL, "workspace too small: need " + std::to_string(need) + " bytes");
    return decode_launch(h, d->q, d->dtype, d->batch, d->hq, d->hkv, d->k, d->v, d->seq_len, d->max_T, d->scale,
                         d->logits, d->out, d->workspace, ns, chunk, stream, x);
}

int kvq_decode_attend_noalloc(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv,
                              const kvq_cache* k, const kvq_cache* v, const int32_t* seq_len, int64_t max_T,
                              float scale, float* logits, float* out, void* stream) {
    g_err.clear();
    int ns = 0;
    int64_t chunk = 0;
    size_t need = 0;
    if (int e = decode_check(h, dtype, batch, hq, hkv, k, v, q, seq_len, max_T, scale, out, &ns, &chunk, &need))
        return e;
    if (need > kvq::kNoAllocScratchBytes)
        return fail(KVQ_EINVAL, "these sizes need " + std::to_string(need) + " bytes of decode scratch, more than the " +
                                    std::to_string(kvq::kNoAllocScratchBytes) +
                                    " bytes built into the library; use kvq_decode_attend with a workspace");
    // check_handle (in decode_check) made sure h->device is current; the
    // scratch address is looked up for, and cached under, the current device.
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device)
        return fail(KVQ_EINVAL, "the handle's device is not the current device");
    void* scratch = nullptr;
    const cudaError_t e = kvq::noalloc_scratch(cur, &scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the decode scratch");
    return decode_launch(h, q, dtype, batch, hq, hkv, k, v, seq_len, max_T, scale, logits, out, scratch, ns, chunk,
                         stream);
}

int kvq_probe_wait_timeout(kvq_handle h, uint32_t polls, void* stream) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    if (polls == 0 || polls > (1u << 20)) return fail(KVQ_EINVAL, "polls must be in 1..2^20");
    const cudaError_t e = kvq::launch_wait_timeout_probe(h->d_status, polls, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "wait-timeout probe launch");
    return KVQ_OK;
}

int kvq_status(kvq_handle h, void* stream, uint32_t* bits) {
    g_err.clear();
    if (int e = check_handle(h)) return e;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(&v, h->d_status, sizeof(v), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(h->d_status, 0, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "kvq_status");
    if (bits) *bits = v;
    if (v & KVQ_STATUS_TIMEOUT) return fail(KVQ_ETIMEOUT, "a kernel's bounded wait gave up");
    if (v & (KVQ_STATUS_NONFINITE | KVQ_STATUS_NORM_OVERFLOW))
        return fail(KVQ_ENONFINITE, "non-finite input or a norm above the fp16 range");
    return KVQ_OK;
}

}  // extern "C"
