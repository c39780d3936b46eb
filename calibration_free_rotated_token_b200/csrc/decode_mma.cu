// decode_mma.cu -- decode attention on the tensor cores (warp-level int8
// MMA), for 1- and 2-bit codebooks.
//
// Method (TurboQuant blog, "Como Implementar": the query is rotated once and
// the logits come straight from the stored indices; PolarQuant section 2:
// dequantisation by centroids, inverse rotation and the stored norm):
//   l_t = scale (n_t/d) ( <q', c[code_t]> + sqrt(pi/2)/m gamma_t <p, 2 bit_t - 1> )
//   A   = sum_t w_t n_t c[vcode_t],  B = sum_t w_t n_t gamma_t (2 vbit_t - 1)
// with w the softmax weights (running max, exact merge of the splits).
//
// Design (sm_100a, one GPU):
// * A symmetric codebook of 2^b <= 4 levels is affine in the stored bit
//   planes: c[code] = c0 + (c1 - c0) bit0 + (c2 - c0) bit1 (the bit0*bit1
//   coefficient c3 - c2 - c1 + c0 vanishes by symmetry).  So every dot
//   product above is a constant plus plain sums of 0/1 planes, and both
//   contractions run as exact integer tensor-core products:
//   - keys: D(16 tokens x 8) += A(16 tokens x 32 coords, 0/1) B(32 coords x 8)
//     where B holds the query (times the plane coefficient) as three signed
//     8-bit digits per head (21-bit fixed point);
//   - values: D(16 x 8 coords) += A(16 x 32 tokens) B(32 tokens x 8 coords,
//     0/1) where A holds the softmax weights as three 8-bit digits per head.
// * The 0/1 operands come straight from the packed words: one shift and one
//   mask give four elements (bits t, t+8, t+16, t+24 of a word), so keys read
//   one record per token and values read the block-32 layout (bits of 32
//   tokens of one coordinate in a word).  The K-element order this implies is
//   folded into the precomputed query fragments and the weight fragments.
// * Per CTA: one (split, KV head, sequence); 256-token sub-chunks staged by
//   1-D bulk copies into double-buffered shared memory; phase K (logits),
//   phase S (softmax statistics, weight digits), phase V (value sums, int32
//   per sub-chunk, merged into fp32 with the running-max rescale).
// * Every mbarrier wait is bounded; all threads take the same decision.
#include <cfloat>

#include "kvq_internal.h"
#include "sm100.cuh"

namespace kvq {

namespace {

constexpr int kThreads = 128;                           // 4 warps
constexpr float kSqrtHalfPi = 1.2533141373155002512f;  // sqrt(pi/2)
constexpr float kDigitRange = 2.0e6f;                   // |X| <= 2e6 < 2^21: three balanced int8 digits

template <int D>
struct DTile {
    static constexpr int TC = (D == 256) ? 128 : 256;  // tokens per sub-chunk
};

// Balanced base-128 digits of an integer |X| <= kDigitRange: X = d0 2^14 + d1 2^7 + d2.
__device__ __forceinline__ void digits3(int X, int& d0, int& d1, int& d2) {
    d2 = ((X + 64) & 127) - 64;
    const int X1 = (X - d2) >> 7;
    d1 = ((X1 + 64) & 127) - 64;
    d0 = (X1 - d1) >> 7;
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
           ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

__device__ __forceinline__ float sign_of(const uint32_t* pair_sign, int j) {
    return ((pair_sign[j >> 1] >> ((j & 1) ? 31 : 15)) & 1u) ? -1.f : 1.f;
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i) {
    if (DT == 0) return reinterpret_cast<const float*>(p)[i];
    if (DT == 1) return __half2float(reinterpret_cast<const __half*>(p)[i]);
    const uint16_t u = reinterpret_cast<const uint16_t*>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Key-side column map of the query fragments: n-tile nt, column n -> (head,
// digit) or -1 for padding.  With G <= 4 thread t of the MMA ends up with
// head t (columns 2t, 2t+1 of n-tile 0 = digits 0, 1; column 2t of n-tile 1 =
// digit 2); with G = 8 it gets heads t and t+4.
template <int G>
__device__ __forceinline__ int key_col_head(int nt, int n, int* dig) {
    if (G <= 4) {
        if (nt == 0) { *dig = n & 1; return n >> 1; }
        if (n & 1) return -1;
        *dig = 2;
        return n >> 1;
    } else {
        if (nt < 2) { *dig = n & 1; return (n >> 1) + 4 * nt; }
        *dig = 2;
        return (n >> 1) + 4 * (n & 1);
    }
}

// Query preparation for one (sequence, KV head) group: q' = H (delta .* q),
// p = S q' per query head, the three-digit fixed-point fragments of
// coef_P q' (code planes) and p (QJL rows) in MMA B-fragment order, and the
// per-head scalars {c0 sum q', sigma_code, sigma_qjl, sum p}.
template <int D, int B, bool QJL, int G, int DT>
__global__ void __launch_bounds__(kThreads) qfrag_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int M = D;
    constexpr int NTK = (G <= 4) ? 2 : 3;
    constexpr int KS = (B + (QJL ? 1 : 0)) * (D / 32);
    __shared__ float sq[G][D];
    __shared__ float sp[G][QJL ? M : 1];
    __shared__ float ssig[G][2];
    const int hk = blockIdx.x % a.hkv, bi = blockIdx.x / a.hkv;
    const int64_t qh0 = static_cast<int64_t>(bi) * a.hq + static_cast<int64_t>(hk) * G;
    const int tid = threadIdx.x;
    for (int e = tid; e < G * D; e += kThreads) {
        const int h = e / D, j = e % D;
        sq[h][j] = sign_of(a.pair_sign, j) * load_elem<DT>(a.q, (qh0 + h) * D + j);
    }
    __syncthreads();
    // FWHT of every head in shared memory
    for (int hs = 1; hs < D; hs <<= 1) {
        for (int e = tid; e < G * D / 2; e += kThreads) {
            const int h = e / (D / 2), pp = e % (D / 2);
            const int i = (pp / hs) * 2 * hs + (pp % hs);
            const float x = sq[h][i], y = sq[h][i + hs];
            sq[h][i] = x + y;
            sq[h][i + hs] = x - y;
        }
        __syncthreads();
    }
    if (QJL) {
        for (int e = tid; e < G * M; e += kThreads) {
            const int h = e / M, i = e % M;
            const __half* Si = a.S + static_cast<int64_t>(i) * D;
            float acc = 0.f;
            for (int j = 0; j < D; ++j) acc = fmaf(__half2float(Si[j]), sq[h][j], acc);
            sp[h][i] = acc;
        }
        __syncthreads();
    }
    // plane coefficients: c[code] = c0 + coef0 bit0 (+ coef1 bit1)
    const float c0 = a.centroid[0];
    const float coef0 = a.centroid[1] - c0;
    const float coef1 = (B == 2) ? a.centroid[2] - c0 : 0.f;
    const float cmax = fmaxf(fabsf(coef0), fabsf(coef1));
    // one warp per head: max |q'|, max |p|, sums
    for (int h = tid / 32; h < G; h += kThreads / 32) {
        const int ln = tid % 32;
        float mq = 0.f, mp = 0.f, s_q = 0.f, s_p = 0.f;
        for (int j = ln; j < D; j += 32) {
            mq = fmaxf(mq, fabsf(sq[h][j]));
            s_q += sq[h][j];
            if (QJL) {
                mp = fmaxf(mp, fabsf(sp[h][j]));
                s_p += sp[h][j];
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            mq = fmaxf(mq, __shfl_xor_sync(0xFFFFFFFFu, mq, o));
            mp = fmaxf(mp, __shfl_xor_sync(0xFFFFFFFFu, mp, o));
            s_q += __shfl_xor_sync(0xFFFFFFFFu, s_q, o);
            s_p += __shfl_xor_sync(0xFFFFFFFFu, s_p, o);
        }
        if (ln == 0) {
            const float sig_c = (mq * cmax > 0.f) ? mq * cmax / kDigitRange : 1.f;
            const float sig_q = (mp > 0.f) ? mp / kDigitRange : 1.f;
            ssig[h][0] = sig_c;
            ssig[h][1] = sig_q;
            a.qscal[(qh0 + h) * 4 + 0] = c0 * s_q;
            a.qscal[(qh0 + h) * 4 + 1] = sig_c;
            a.qscal[(qh0 + h) * 4 + 2] = sig_q;
            a.qscal[(qh0 + h) * 4 + 3] = s_p;
        }
    }
    __syncthreads();
    // B fragments: [k-step][n-tile][lane] of (b0, b1)
    uint2* frag = a.qfrag + static_cast<int64_t>(blockIdx.x) * KS * NTK * 32;
    for (int e = tid; e < KS * NTK * 32; e += kThreads) {
        const int lane = e % 32, nt = (e / 32) % NTK, ks = e / (32 * NTK);
        const int g = lane >> 2, t = lane & 3;
        int dig = 0;
        const int h = key_col_head<G>(nt, g, &dig);
        uint32_t b[2] = {0u, 0u};
        if (h >= 0 && h < G) {
            const int plane = ks / (D / 32), w = ks % (D / 32);
            const bool is_q = plane >= B;
            const float coef = (plane == 0) ? coef0 : coef1;
            const float sig = is_q ? ssig[h][1] : ssig[h][0];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                int dd[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = 32 * w + t + 4 * half + 8 * i;
                    const float v = is_q ? sp[h][j] : coef * sq[h][j];
                    const int X = __float2int_rn(v / sig);
                    int d0, d1, d2;
                    digits3(X, d0, d1, d2);
                    dd[i] = dig == 0 ? d0 : (dig == 1 ? d1 : d2);
                }
                b[half] = pack4(dd[0], dd[1], dd[2], dd[3]);
            }
        }
        frag[e] = make_uint2(b[0], b[1]);
    }
}

// Shared-memory plan of the split kernel.
template <int D, int B, bool QJL, int G>
struct MmaSmem {
    static constexpr int M = D;
    static constexpr int TC = DTile<D>::TC;
    static constexpr int NTK = (G <= 4) ? 2 : 3;
    static constexpr int RT = (G <= 4) ? 1 : 2;
    static constexpr int KS = (B + (QJL ? 1 : 0)) * (D / 32);
    static constexpr int GP = (G <= 4) ? 4 : 8;            // heads incl. padding
    // staging of one sub-chunk
    static constexpr int kKc = TC * B * D / 8;             // key codes (token layout)
    static constexpr int kKq = QJL ? TC * M / 8 : 0;       // key sign bits
    static constexpr int kKn = TC * 4;                     // key norms
    static constexpr int kVc = (TC / 32) * B * D * 4;      // value codes (block-32)
    static constexpr int kVq = QJL ? (TC / 32) * M * 4 : 0;
    static constexpr int kVn = TC * 4;
    static constexpr int kStage = kKc + kKq + kKn + kVc + kVq + kVn;
    static constexpr int kFrag = KS * NTK * 32 * 8;        // query fragments
    static constexpr int kLog = GP * TC * 4;               // logits of the sub-chunk
    static constexpr int kWfrag = (TC / 32) * RT * 32 * 16;  // weight digits, per kind
    static constexpr int kBytes = 2 * kStage + kFrag + kLog + 2 * kWfrag + 1024;
};

template <int D, int B, bool QJL, int G>
__global__ void __launch_bounds__(kThreads) decode_mma_kernel(const __grid_constant__ DecodeArgs a) {
    using L = MmaSmem<D, B, QJL, G>;
    constexpr int M = D, TC = L::TC, NTK = L::NTK, RT = L::RT, KS = L::KS, GP = L::GP;
    constexpr int KWT = B * D / 32;           // code words per token (key layout)
    constexpr int QWT = QJL ? M / 32 : 0;     // sign words per token
    constexpr int NTV = D / 32;               // value n-tiles per warp and plane (D/4 coordinates / 8)
    constexpr int NPV = B + (QJL ? 1 : 0);
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* stage[2] = {smem, smem + L::kStage};
    uint2* sfrag = reinterpret_cast<uint2*>(smem + 2 * L::kStage);
    float* slog = reinterpret_cast<float*>(smem + 2 * L::kStage + L::kFrag);  // [GP][TC]
    uint32_t* swc = reinterpret_cast<uint32_t*>(smem + 2 * L::kStage + L::kFrag + L::kLog);  // code-weight digits
    uint32_t* swq = swc + L::kWfrag / 4;                                                       // QJL-weight digits
    uint8_t* misc = smem + 2 * L::kStage + L::kFrag + L::kLog + 2 * L::kWfrag;
    uint64_t* bar = reinterpret_cast<uint64_t*>(misc);      // [2]
    float* sred = reinterpret_cast<float*>(misc + 16);      // [4 warps][GP][3]
    float* shead = sred + 4 * GP * 3;                        // [GP][8]: scalars, running state

    const int split = blockIdx.x, hk = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int64_t T = min(static_cast<int64_t>(max(a.seq_len[bi], 0)), a.max_T);
    const int64_t t0 = static_cast<int64_t>(split) * a.chunk;
    const int64_t t1e = min(t0 + a.chunk, a.max_T);
    const int64_t t1 = min(t1e, T);
    const int64_t stream = static_cast<int64_t>(bi) * a.hkv + hk;
    const int64_t qh0 = static_cast<int64_t>(bi) * a.hq + static_cast<int64_t>(hk) * G;
    const int64_t grp = static_cast<int64_t>(bi) * a.hkv + hk;

    // stream bases
    const uint8_t* kc = reinterpret_cast<const uint8_t*>(a.kcodes) + stream * a.kcap * (B * D / 8);
    const uint8_t* kq = QJL ? reinterpret_cast<const uint8_t*>(a.kqjl) + stream * a.kcap * (M / 8) : nullptr;
    const uint8_t* kn = reinterpret_cast<const uint8_t*>(a.knorms) + stream * a.kcap * 4;
    const uint8_t* vc = reinterpret_cast<const uint8_t*>(a.vcodes) + stream * (a.vcap / 32) * B * D * 4;
    const uint8_t* vq = QJL ? reinterpret_cast<const uint8_t*>(a.vqjl) + stream * (a.vcap / 32) * M * 4 : nullptr;
    const uint8_t* vn = reinterpret_cast<const uint8_t*>(a.vnorms) + stream * a.vcap * 4;

    // ---- set-up: query fragments, per-head scalars, zero weight digits, barriers
    {
        const uint2* gf = a.qfrag + grp * KS * NTK * 32;
        for (int e = tid; e < KS * NTK * 32; e += kThreads) sfrag[e] = gf[e];
        for (int e = tid; e < 2 * L::kWfrag / 4; e += kThreads) swc[e] = 0u;
        if (tid < GP) {
            float* hs = shead + tid * 8;
            if (tid < G) {
                const float* qs = a.qscal + (qh0 + tid) * 4;
                hs[0] = qs[0]; hs[1] = qs[1]; hs[2] = qs[2]; hs[3] = qs[3];
            } else {
                hs[0] = hs[1] = hs[2] = hs[3] = 0.f;
            }
            hs[4] = -INFINITY;  // running max
            hs[5] = 0.f;        // running sum of exp
            hs[6] = 0.f;        // running sum of code weights (Omega)
            hs[7] = 0.f;        // running sum of QJL weights (Omega')
        }
        if (tid == 0) {
            mbar_init(&bar[0], 1);
            mbar_init(&bar[1], 1);
            fence_mbar_init();
        }
    }
    __syncthreads();

    const int nsub = static_cast<int>((t1e - t0 + TC - 1) / TC);
    // tokens of the sub-chunk that exist in the cache (rounded to whole blocks of 32)
    auto issue = [&](int sc) {
        const int64_t tb = t0 + static_cast<int64_t>(sc) * TC;
        const int64_t have = min(static_cast<int64_t>(TC), t1 - tb);
        if (have <= 0) return false;
        const int64_t nt = (have + 31) / 32 * 32;  // <= capacity - tb (capacity is a multiple of 32)
        uint8_t* st = stage[sc & 1];
        uint64_t* b = &bar[sc & 1];
        const uint32_t bytes = static_cast<uint32_t>(nt * (B * D / 8 + (QJL ? M / 8 : 0) + 4) +
                                                     (nt / 32) * (B * D * 4 + (QJL ? M * 4 : 0)) + nt * 4);
        mbar_arrive_expect_tx(b, bytes);
        bulk_load(st, kc + tb * (B * D / 8), static_cast<uint32_t>(nt * (B * D / 8)), b);
        if (QJL) bulk_load(st + L::kKc, kq + tb * (M / 8), static_cast<uint32_t>(nt * (M / 8)), b);
        bulk_load(st + L::kKc + L::kKq, kn + tb * 4, static_cast<uint32_t>(nt * 4), b);
        bulk_load(st + L::kKc + L::kKq + L::kKn, vc + (tb / 32) * B * D * 4, static_cast<uint32_t>((nt / 32) * B * D * 4),
                  b);
        if (QJL)
            bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc, vq + (tb / 32) * M * 4,
                      static_cast<uint32_t>((nt / 32) * M * 4), b);
        bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq, vn + tb * 4, static_cast<uint32_t>(nt * 4), b);
        return true;
    };
    bool armed0 = false, armed1 = false;
    if (tid == 0) {
        armed0 = issue(0);
        armed1 = nsub > 1 ? issue(1) : false;
    }
    uint32_t phase[2] = {0u, 0u};
    bool alive = true;

    // fp32 running value sums: this thread's coordinates of warp `warp`
    // (code part combined over planes; QJL part), head g (G <= 4, lanes g < 4)
    // or head g (G = 8, all lanes).
    float accA[NTV][2], accB[NTV][2];
#pragma unroll
    for (int nt = 0; nt < NTV; ++nt) accA[nt][0] = accA[nt][1] = accB[nt][0] = accB[nt][1] = 0.f;

    const float kappa = kSqrtHalfPi / M;
    const float coef0 = a.centroid[1] - a.centroid[0];
    const float coef1 = (B == 2) ? a.centroid[2] - a.centroid[0] : 0.f;

    for (int sc = 0; sc < nsub; ++sc) {
        const int64_t tb = t0 + static_cast<int64_t>(sc) * TC;
        const int64_t have = min(static_cast<int64_t>(TC), t1 - tb);  // may be <= 0 (split past the context)
        const uint8_t* st = stage[sc & 1];
        if (have > 0) {
            const bool ok = mbar_wait(&bar[sc & 1], phase[sc & 1], a.status);
            phase[sc & 1] ^= 1u;
            if (__syncthreads_or(!ok)) { alive = false; break; }
        }
        const uint32_t* sKc = reinterpret_cast<const uint32_t*>(st);
        const uint32_t* sKq = reinterpret_cast<const uint32_t*>(st + L::kKc);
        const __half2* sKn = reinterpret_cast<const __half2*>(st + L::kKc + L::kKq);
        const uint32_t* sVc = reinterpret_cast<const uint32_t*>(st + L::kKc + L::kKq + L::kKn);
        const uint32_t* sVq = reinterpret_cast<const uint32_t*>(st + L::kKc + L::kKq + L::kKn + L::kVc);
        const __half2* sVn = reinterpret_cast<const __half2*>(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq);

        // ---------------- phase K: logits of the sub-chunk ----------------
        for (int mt = warp; mt < TC / 16; mt += 4) {
            const int tl0 = mt * 16 + g, tl1 = tl0 + 8;
            int accc[NTK][4], accq[NTK][4];
#pragma unroll
            for (int nt = 0; nt < NTK; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) accc[nt][r] = accq[nt][r] = 0;
            if (tb + mt * 16 < t1) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const bool is_q = ks >= B * (D / 32);
                    uint32_t w0, w1;
                    if (!is_q) {
                        w0 = sKc[tl0 * KWT + ks];
                        w1 = sKc[tl1 * KWT + ks];
                    } else {
                        w0 = sKq[tl0 * QWT + (ks - B * (D / 32))];
                        w1 = sKq[tl1 * QWT + (ks - B * (D / 32))];
                    }
                    const uint32_t af[4] = {(w0 >> t) & 0x01010101u, (w1 >> t) & 0x01010101u,
                                            (w0 >> (t + 4)) & 0x01010101u, (w1 >> (t + 4)) & 0x01010101u};
#pragma unroll
                    for (int nt = 0; nt < NTK; ++nt) {
                        const uint2 bq = sfrag[(ks * NTK + nt) * 32 + lane];
                        if (!is_q) mma_s8_16832(accc[nt], af, bq.x, bq.y);
                        else mma_s8_16832(accq[nt], af, bq.x, bq.y);
                    }
                }
            }
            // epilogue: thread t owns head t (and t + 4 when G = 8)
#pragma unroll
            for (int hh = 0; hh < (G == 8 ? 2 : 1); ++hh) {
                const int h = t + 4 * hh;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int tl = rr ? tl1 : tl0;
                    const int64_t tg = tb + tl;
                    float l = -INFINITY;
                    if (h < G && tg < t1) {
                        int ci, qi;
                        if (G <= 4) {
                            ci = accc[0][2 * rr] * 16384 + accc[0][2 * rr + 1] * 128 + accc[1][2 * rr];
                            qi = accq[0][2 * rr] * 16384 + accq[0][2 * rr + 1] * 128 + accq[1][2 * rr];
                        } else {
                            ci = accc[hh][2 * rr] * 16384 + accc[hh][2 * rr + 1] * 128 + accc[2][2 * rr + hh];
                            qi = accq[hh][2 * rr] * 16384 + accq[hh][2 * rr + 1] * 128 + accq[2][2 * rr + hh];
                        }
                        const float* hs = shead + h * 8;
                        const float2 nk = __half22float2(sKn[tl]);
                        float dot = hs[0] + hs[1] * static_cast<float>(ci);
                        if (QJL) dot += kappa * nk.y * (2.f * hs[2] * static_cast<float>(qi) - hs[3]);
                        l = a.scale * (nk.x / D) * dot;
                    }
                    if (h < GP) slog[h * TC + tl] = l;
                    if (a.logits != nullptr && h < G && tg < t1e) a.logits[(qh0 + h) * a.max_T + tg] = l;
                }
            }
        }
        __syncthreads();

        // ---------------- phase S: softmax statistics and weight digits ----------------
        // pass 1: per head, the max logit and the max of l + log(n) (and of
        // l + log(n gamma)): the largest weight of the sub-chunk, which sets
        // the scale of its weight digits (so that small weights keep their
        // resolution when the sub-chunk sits far below the running max).
        {
            float mx[GP], mw[GP], mq[GP];
#pragma unroll
            for (int h = 0; h < GP; ++h) mx[h] = mw[h] = mq[h] = -INFINITY;
            for (int tl = tid; tl < TC; tl += kThreads) {
                if (tb + tl < t1) {
                    const float2 nv = __half22float2(sVn[tl]);
                    const float ln = __logf(nv.x), lg = __logf(nv.x * nv.y);
#pragma unroll
                    for (int h = 0; h < GP; ++h) {
                        const float l = slog[h * TC + tl];
                        mx[h] = fmaxf(mx[h], l);
                        mw[h] = fmaxf(mw[h], l + ln);
                        mq[h] = fmaxf(mq[h], l + lg);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], o));
                    mw[h] = fmaxf(mw[h], __shfl_xor_sync(0xFFFFFFFFu, mw[h], o));
                    mq[h] = fmaxf(mq[h], __shfl_xor_sync(0xFFFFFFFFu, mq[h], o));
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    sred[(warp * GP + h) * 3 + 0] = mx[h];
                    sred[(warp * GP + h) * 3 + 1] = mw[h];
                    sred[(warp * GP + h) * 3 + 2] = mq[h];
                }
            }
        }
        __syncthreads();
        // per-head new running max, rescale factor and weight-digit scales
        float* sstat = shead + GP * 8;  // [GP][4]: mnew, alpha, sig_w, sig_wq
        if (tid < GP) {
            const int h = tid;
            float mx = -INFINITY, mw = -INFINITY, mq = -INFINITY;
            for (int w = 0; w < 4; ++w) {
                mx = fmaxf(mx, sred[(w * GP + h) * 3 + 0]);
                mw = fmaxf(mw, sred[(w * GP + h) * 3 + 1]);
                mq = fmaxf(mq, sred[(w * GP + h) * 3 + 2]);
            }
            float* hs = shead + h * 8;
            const float mold = hs[4];
            const float mnew = fmaxf(mold, mx);
            const float alpha = (mnew == -INFINITY) ? 1.f : __expf(mold - mnew);
            hs[4] = mnew;
            const float wmax = (mw == -INFINITY) ? 0.f : __expf(mw - mnew);
            const float qmax = (mq == -INFINITY) ? 0.f : __expf(mq - mnew);
            sstat[h * 4 + 0] = mnew;
            sstat[h * 4 + 1] = alpha;
            sstat[h * 4 + 2] = wmax > 0.f ? wmax / kDigitRange : 1.f;
            sstat[h * 4 + 3] = qmax > 0.f ? qmax / kDigitRange : 1.f;
        }
        __syncthreads();
        // pass 2: weight digits into A-fragment order; sums of exp and weights
        {
            float sum_e[GP], sum_w[GP], sum_wq[GP];
#pragma unroll
            for (int h = 0; h < GP; ++h) sum_e[h] = sum_w[h] = sum_wq[h] = 0.f;
            for (int tl = tid; tl < TC; tl += kThreads) {
                const bool valid = tb + tl < t1;
                const float2 nv = valid ? __half22float2(sVn[tl]) : make_float2(0.f, 0.f);
                // K-element of token u in its block: u = t' + 8 i (+4 for the second half)
                const int u = tl & 31, bb = tl >> 5;
                const int tp = u & 3, half = (u >> 2) & 1, i = u >> 3;
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    float wc = 0.f, wq = 0.f;
                    if (valid && h < G) {
                        const float e = __expf(slog[h * TC + tl] - sstat[h * 4 + 0]);
                        sum_e[h] += e;
                        wc = e * nv.x;
                        wq = wc * nv.y;
                        sum_w[h] += wc;
                        sum_wq[h] += wq;
                    }
                    int dc[3], dq[3];
                    const int xc = min(__float2int_rn(wc / sstat[h * 4 + 2]), static_cast<int>(kDigitRange) + 4096);
                    const int xq = min(__float2int_rn(wq / sstat[h * 4 + 3]), static_cast<int>(kDigitRange) + 4096);
                    digits3(xc, dc[0], dc[1], dc[2]);
                    digits3(xq, dq[0], dq[1], dq[2]);
#pragma unroll
                    for (int dg = 0; dg < 3; ++dg) {
                        // row r of the weight operand: G <= 4: r = h + 4 dg (one row tile);
                        // G = 8: r = h + 8 dg (rows 16..23 -> second row tile)
                        const int r = (G <= 4) ? h + 4 * dg : h + 8 * dg;
                        const int rt = r >> 4, rl = r & 15;
                        const int ln = 4 * (rl & 7) + tp;
                        const int reg = (rl >> 3) + 2 * half;
                        const int byte = ((((bb * RT + rt) * 32 + ln) * 4 + reg) << 2) + i;
                        reinterpret_cast<uint8_t*>(swc)[byte] = static_cast<uint8_t>(dc[dg]);
                        if (QJL) reinterpret_cast<uint8_t*>(swq)[byte] = static_cast<uint8_t>(dq[dg]);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    sum_e[h] += __shfl_xor_sync(0xFFFFFFFFu, sum_e[h], o);
                    sum_w[h] += __shfl_xor_sync(0xFFFFFFFFu, sum_w[h], o);
                    sum_wq[h] += __shfl_xor_sync(0xFFFFFFFFu, sum_wq[h], o);
                }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    sred[(warp * GP + h) * 3 + 0] = sum_e[h];
                    sred[(warp * GP + h) * 3 + 1] = sum_w[h];
                    sred[(warp * GP + h) * 3 + 2] = sum_wq[h];
                }
        }
        __syncthreads();
        if (tid < GP) {
            const int h = tid;
            float te = 0.f, tw = 0.f, twq = 0.f;
            for (int w = 0; w < 4; ++w) {
                te += sred[(w * GP + h) * 3 + 0];
                tw += sred[(w * GP + h) * 3 + 1];
                twq += sred[(w * GP + h) * 3 + 2];
            }
            float* hs = shead + h * 8;
            const float alpha = sstat[h * 4 + 1];
            hs[5] = hs[5] * alpha + te;
            hs[6] = hs[6] * alpha + tw;
            hs[7] = hs[7] * alpha + twq;
        }

        // ---------------- phase V: value sums of the sub-chunk ----------------
        {
            int accv[NPV][NTV][RT][4];
#pragma unroll
            for (int p = 0; p < NPV; ++p)
#pragma unroll
                for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) accv[p][nt][rt][r] = 0;
            const int nblk = have > 0 ? static_cast<int>((have + 31) / 32) : 0;
            for (int bb = 0; bb < nblk; ++bb) {
                uint32_t aw[RT][4], aq[RT][4];
#pragma unroll
                for (int rt = 0; rt < RT; ++rt) {
                    const uint4 x = reinterpret_cast<const uint4*>(swc)[(bb * RT + rt) * 32 + lane];
                    aw[rt][0] = x.x; aw[rt][1] = x.y; aw[rt][2] = x.z; aw[rt][3] = x.w;
                    if (QJL) {
                        const uint4 y = reinterpret_cast<const uint4*>(swq)[(bb * RT + rt) * 32 + lane];
                        aq[rt][0] = y.x; aq[rt][1] = y.y; aq[rt][2] = y.z; aq[rt][3] = y.w;
                    }
                }
#pragma unroll
                for (int p = 0; p < NPV; ++p) {
#pragma unroll
                    for (int nt = 0; nt < NTV; ++nt) {
                        const int coord = warp * (D / 4) + nt * 8 + g;
                        const uint32_t wv = (p < B) ? sVc[(bb * B + p) * D + coord] : sVq[bb * M + coord];
                        const uint32_t b0 = (wv >> t) & 0x01010101u, b1 = (wv >> (t + 4)) & 0x01010101u;
#pragma unroll
                        for (int rt = 0; rt < RT; ++rt) {
                            if (p < B) mma_s8_16832(accv[p][nt][rt], aw[rt], b0, b1);
                            else mma_s8_16832(accv[p][nt][rt], aq[rt], b0, b1);
                        }
                    }
                }
            }
            // merge into the fp32 running sums (rescaled by alpha of this sub-chunk)
#pragma unroll
            for (int nt = 0; nt < NTV; ++nt) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    int vi[NPV];
                    int head;
#pragma unroll
                    for (int p = 0; p < NPV; ++p) {
                        if (G <= 4) {
                            // rows g (digit 0 or 1, head g & 3) and g + 8 (digit 2 or pad)
                            const int d1 = __shfl_xor_sync(0xFFFFFFFFu, accv[p][nt][0][c], 16);
                            vi[p] = accv[p][nt][0][c] * 16384 + d1 * 128 + accv[p][nt][0][2 + c];
                        } else {
                            vi[p] = accv[p][nt][0][c] * 16384 + accv[p][nt][0][2 + c] * 128 + accv[p][nt][1][c];
                        }
                    }
                    head = g;
                    const bool own = (G <= 4) ? (g < 4) : true;
                    if (own && head < G) {
                        const float alpha = sstat[head * 4 + 1];
                        const float sgw = sstat[head * 4 + 2], sgq = sstat[head * 4 + 3];
                        float code = coef0 * static_cast<float>(vi[0]);
                        if (B == 2) code += coef1 * static_cast<float>(vi[1 % NPV]);
                        accA[nt][c] = accA[nt][c] * alpha + sgw * code;
                        if (QJL) accB[nt][c] = accB[nt][c] * alpha + sgq * 2.f * static_cast<float>(vi[NPV - 1]);
                    }
                }
            }
        }
        __syncthreads();  // stage and weight digits are reused by the next sub-chunk
        if (tid == 0 && sc + 2 < nsub) {
            if (sc & 1) armed1 = issue(sc + 2);
            else armed0 = issue(sc + 2);
        }
    }
    if (tid == 0) {
        // loads in flight are waited for before exit (only when a wait gave up)
        if (!alive) {
            if (armed0) mbar_wait(&bar[0], phase[0], a.status);
            if (armed1) mbar_wait(&bar[1], phase[1], a.status);
        }
    }

    // ---------------- partials: {M, L, A[D], B[M]} per query head ----------------
    constexpr int PART = 2 + D + M;
    const bool own = (G <= 4) ? (g < 4) : true;
    const int head = g;
    if (own && head < G) {
        float* pp = a.part + ((qh0 + head) * a.nsplit + split) * PART;
        const float* hs = shead + head * 8;
        const float c0 = a.centroid[0];
#pragma unroll
        for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int coord = warp * (D / 4) + nt * 8 + 2 * t + c;
                pp[2 + coord] = c0 * hs[6] + accA[nt][c];
                if (QJL) pp[2 + D + coord] = accB[nt][c] - hs[7];
            }
    }
    if (tid < G) {
        float* pp = a.part + ((qh0 + tid) * a.nsplit + split) * PART;
        pp[0] = shead[tid * 8 + 4];
        pp[1] = shead[tid * 8 + 5];
    }
}

}  // namespace

template <int D, int B, bool QJL, int G>
static cudaError_t launch_mma_g(const DecodeArgs& a, cudaStream_t s) {
    const int groups = a.batch * a.hkv;
    switch (a.qdtype) {
        case 0: qfrag_kernel<D, B, QJL, G, 0><<<groups, kThreads, 0, s>>>(a); break;
        case 1: qfrag_kernel<D, B, QJL, G, 1><<<groups, kThreads, 0, s>>>(a); break;
        default: qfrag_kernel<D, B, QJL, G, 2><<<groups, kThreads, 0, s>>>(a); break;
    }
    using L = MmaSmem<D, B, QJL, G>;
    auto kern = decode_mma_kernel<D, B, QJL, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.nsplit, a.hkv, a.batch), kThreads, L::kBytes, s>>>(a);
    return cudaGetLastError();
}

template <int D, int B, bool QJL>
static cudaError_t launch_mma_d(const DecodeArgs& a, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_mma_g<D, B, QJL, 1>(a, s);
        case 2: return launch_mma_g<D, B, QJL, 2>(a, s);
        case 4: return launch_mma_g<D, B, QJL, 4>(a, s);
        default: return launch_mma_g<D, B, QJL, 8>(a, s);
    }
}

// Query fragments + split kernel of the tensor-core path (b <= 2).
cudaError_t launch_decode_mma(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s) {
    const bool qjl = (h->flags & 1u) != 0;
#define KVQ_MMA_CASE(D_, B_)                                                                              \
    if (h->d == D_ && h->b == B_)                                                                         \
        return qjl ? launch_mma_d<D_, B_, true>(a, s) : launch_mma_d<D_, B_, false>(a, s);
    KVQ_MMA_CASE(64, 1) KVQ_MMA_CASE(64, 2) KVQ_MMA_CASE(128, 1) KVQ_MMA_CASE(128, 2) KVQ_MMA_CASE(256, 1)
    KVQ_MMA_CASE(256, 2)
#undef KVQ_MMA_CASE
    return cudaErrorNotSupported;
}

size_t decode_mma_qfrag_bytes(const kvq_ctx* h, int G) {
    const int NTK = (G <= 4) ? 2 : 3;
    const int KS = (h->b + ((h->flags & 1u) ? 1 : 0)) * (h->d / 32);
    return static_cast<size_t>(KS) * NTK * 32 * 8;
}

}  // namespace kvq
