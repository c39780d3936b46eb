// decode_mma.cu -- decode attention on the tensor cores (warp-level integer
// MMA), for 1- and 2-bit codebooks and 3-bit ones at d <= 128; plain caches
// (with or without QJL) and NSN caches.
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
//   coefficient c3 - c2 - c1 + c0 vanishes by symmetry); a 3-bit one is
//   affine in its three planes plus their parity (PlaneCoefs).  So every dot
//   product above is a constant plus plain sums of 0/1 planes, and both
//   contractions run as exact integer tensor-core products (m16n8k32):
//   - keys:   D(16 tokens x 8) += A(16 tokens x 32 coords) B(32 coords x 8),
//     B = the query (times the plane coefficient) in four signed base-128
//     digits per head;
//   - values: D(16 x 8 coords) += A(16 x 32 tokens) B(32 tokens x 8 coords),
//     A = the softmax weights in four unsigned base-256 digits per head.
// * The 0/1 operand is one AND of a packed word with a per-lane mask: byte
//   i of (w & (0x01010101 << s)) is bit s + 8i of w, valued 2^s.  The
//   factor 2^s is taken out on the other operand, which carries 2^(7 - s)
//   (so every product is 2^7 times the intended one).
// * The weight digits are the four bytes of one integer conversion,
//   round(w 2^(7-s)/sigma) < 2^31 (s = 7 keeps 24 bits of the largest weight
//   of the sub-chunk).
// * A persistent grid walks (stream, split) items; per item, sub-chunks of
//   TC tokens stream through two shared-memory stages by 1-D bulk copies;
//   per sub-chunk: phase K (logits), phase S (softmax statistics and weight
//   digits), phase V (value sums, int32 per sub-chunk, merged into fp32 with
//   the running-max rescale).
// * Every mbarrier wait is bounded; all threads take the same decision.
#include <cfloat>
#include <type_traits>

#include "kvq_internal.h"
#include "sm100.cuh"

namespace kvq {

namespace {

constexpr int kThreads = 128;                           // 4 warps
constexpr float kSqrtHalfPi = 1.2533141373155002512f;  // sqrt(pi/2)
constexpr float kQRange = 1.3e8f;                       // |X| <= 1.3e8: four balanced base-128 digits
constexpr float kWCap = 2.0e9f;                         // weight integers stay below 2^31
constexpr uint32_t kLowBits = 0x01010101u;

template <int D>
struct DTile {
    static constexpr int TC = (D == 256) ? 128 : 256;  // tokens per sub-chunk
};

template <int G>
struct HeadCfg {
    // key n-tiles (4 digit columns per head): G <= 2 takes one n-tile of two
    // heads (column g = head g / 4, digit g % 4), G = 4 two and G = 8 four
    // (column g of n-tile nt = head g / 2 + 4 (nt / 2), digit g % 2 + 2 (nt % 2))
    static constexpr int NTK = (G <= 2) ? 1 : (G <= 4) ? 2 : 4;
    static constexpr int RT = (G <= 4) ? 1 : 2;   // value m-tiles: 4 digit rows per head
    static constexpr int GP = (G <= 4) ? 4 : 8;   // heads incl. padding
    static constexpr int CPL = (G <= 4) ? 1 : 2;  // value columns merged per lane
};

// Balanced base-128 digits of |X| <= kQRange: X = d0 2^21 + d1 2^14 + d2 2^7 + d3.
__device__ __forceinline__ void digits4(int X, int (&d)[4]) {
    d[3] = ((X + 64) & 127) - 64;
    X = (X - d[3]) >> 7;
    d[2] = ((X + 64) & 127) - 64;
    X = (X - d[2]) >> 7;
    d[1] = ((X + 64) & 127) - 64;
    d[0] = (X - d[1]) >> 7;
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

__device__ __forceinline__ float load_elem_rt(const void* p, int dt, int64_t i) {
    if (dt == 0) return reinterpret_cast<const float*>(p)[i];
    const uint16_t u = reinterpret_cast<const uint16_t*>(p)[i];
    return dt == 1 ? __half2float(__ushort_as_half(u)) : __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Warp-level integer products: d(16x8, s32) += a(16x32, u8, row) * b(32x8, s8 or u8, col).
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
}
// Operand quads as uint4 / pairs as uint2 (lets the allocator keep them in
// aligned register groups).
__device__ __forceinline__ void mma_u8s8_q(int (&d)[4], uint4 a, uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y));
}
__device__ __forceinline__ void mma_u8s8_qz(int (&d)[4], uint4 a, uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(0));
}
__device__ __forceinline__ void mma_u8u8_q(int (&d)[4], uint4 a, uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y));
}
__device__ __forceinline__ void mma_u8u8_qz(int (&d)[4], uint4 a, uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(0));
}

// The same with a zero accumulator input (first K-step of a chain).
__device__ __forceinline__ void mma_u8s8_z(int (&d)[4], const uint32_t (&a)[4], uint2 b) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "r"(0));
}
__device__ __forceinline__ void mma_u8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Query preparation for one (sequence, KV head) group: q' = H (delta .* q),
// p = S q' per query head, the digit fragments of coef_P q' (code planes)
// and p (QJL rows) in MMA B-fragment order, and the per-head scalars
// {c0 sum q', sigma_code/128, sigma_qjl/128, sum p}.
//
// B fragment of lane (g, t) in n-tile nt, K-step ks (32 coordinates 32w ..):
// column g = (head (g >> 1) + 4 (nt >> 1), digit (g & 1) + 2 (nt & 1)); K
// index 4t + i is coordinate 32w + t + 8i with factor 2^(7 - t), K index
// 16 + 4t + i is coordinate 32w + t + 4 + 8i with factor 2^(3 - t).
// Plane form of a symmetric codebook of 2^B levels (B <= 3):
//   c[code] = cst + sum_v coef[v] plane_v(code),
// plane_v = bit v of the code for v < B, and for B = 3 a fourth plane
// bit0 ^ bit1 ^ bit2.  In +-1 variables s_p = 2 bit_p - 1 a codebook with
// c[~k] = -c[k] is an odd function, so its multilinear form has only the odd
// terms: sum_p a_p s_p (B <= 2: exactly the planes), plus a_3 s0 s1 s2 for
// B = 3, and s0 s1 s2 = 2 (bit0 ^ bit1 ^ bit2) - 1.
template <int B>
struct PlaneCoefs {
    static constexpr int PV = (B == 3) ? 4 : B;  // code planes, the parity plane included
    float cst;
    float coef[PV];
};
template <int B>
__device__ __forceinline__ PlaneCoefs<B> plane_coefs(const float* c) {
    PlaneCoefs<B> r;
    if constexpr (B <= 2) {
        r.cst = c[0];
        r.coef[0] = c[1] - c[0];
        if constexpr (B == 2) r.coef[1] = c[2] - c[0];
    } else {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float s0 = (k & 1) ? 1.f : -1.f, s1 = (k & 2) ? 1.f : -1.f, s2 = (k & 4) ? 1.f : -1.f;
            a0 = fmaf(c[k], s0, a0);
            a1 = fmaf(c[k], s1, a1);
            a2 = fmaf(c[k], s2, a2);
            a3 = fmaf(c[k], s0 * s1 * s2, a3);
        }
        r.cst = -0.125f * (a0 + a1 + a2 + a3);
        r.coef[0] = 0.25f * a0;
        r.coef[1] = 0.25f * a1;
        r.coef[2] = 0.25f * a2;
        r.coef[3] = 0.25f * a3;
    }
    return r;
}

template <int D, int B, bool QJL, int G, int DT>
__global__ void __launch_bounds__(kThreads) qfrag_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int M = D;
    constexpr int NTK = HeadCfg<G>::NTK;
    constexpr int PV = PlaneCoefs<B>::PV;
    constexpr int KS = (PV + (QJL ? 1 : 0)) * (D / 32);
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
        // p = S q' for every head of the group: thread i reads row i of S
        // once (16-byte loads, all in flight together) and feeds all G heads.
        for (int i = tid; i < M; i += kThreads) {
            const uint4* Si = reinterpret_cast<const uint4*>(a.S + static_cast<int64_t>(i) * D);
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
            for (int j0 = 0; j0 < D / 8; j0 += 8) {
                uint4 w[8];
#pragma unroll
                for (int u = 0; u < 8 && j0 + u < D / 8; ++u) w[u] = Si[j0 + u];
#pragma unroll
                for (int u = 0; u < 8 && j0 + u < D / 8; ++u) {
                    const __half2* hw = reinterpret_cast<const __half2*>(&w[u]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 sv = __half22float2(hw[k]);
                        const int j = 8 * (j0 + u) + 2 * k;
#pragma unroll
                        for (int h = 0; h < G; ++h) acc[h] = fmaf(sv.y, sq[h][j + 1], fmaf(sv.x, sq[h][j], acc[h]));
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) sp[h][i] = acc[h];
        }
        __syncthreads();
    }
    // plane coefficients: c[code] = cst + sum_v coef[v] plane_v
    const PlaneCoefs<B> pc = plane_coefs<B>(a.centroid);
    const float c0 = pc.cst;
    float cmax = 0.f;
#pragma unroll
    for (int v = 0; v < PV; ++v) cmax = fmaxf(cmax, fabsf(pc.coef[v]));
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
            // X = v 2^(7-s) / sig stays within kQRange for every s
            const float sig_c = (mq * cmax > 0.f) ? mq * cmax * 128.f / kQRange : 1.f;
            const float sig_q = (mp > 0.f) ? mp * 128.f / kQRange : 1.f;
            ssig[h][0] = sig_c;
            ssig[h][1] = sig_q;
            a.qscal[(qh0 + h) * 4 + 0] = c0 * s_q;
            a.qscal[(qh0 + h) * 4 + 1] = sig_c * (1.f / 128.f);
            a.qscal[(qh0 + h) * 4 + 2] = sig_q * (1.f / 128.f);
            a.qscal[(qh0 + h) * 4 + 3] = s_p;
        }
    }
    __syncthreads();
    uint2* frag = a.qfrag + static_cast<int64_t>(blockIdx.x) * KS * NTK * 32;
    for (int e = tid; e < KS * NTK * 32; e += kThreads) {
        const int lane = e % 32, nt = (e / 32) % NTK, ks = e / (32 * NTK);
        const int g = lane >> 2, t = lane & 3;
        const int h = (NTK == 1) ? (g >> 2) : (g >> 1) + 4 * (nt >> 1);
        const int dig = (NTK == 1) ? (g & 3) : (g & 1) + 2 * (nt & 1);
        uint32_t b[2] = {0u, 0u};
        if (h < G) {
            const int plane = ks / (D / 32), w = ks % (D / 32);
            const bool is_q = plane >= PV;
            float coef = 0.f;
#pragma unroll
            for (int v = 0; v < PV; ++v) coef = (plane == v) ? pc.coef[v] : coef;
            const float sig = is_q ? ssig[h][1] : ssig[h][0];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const float fac = static_cast<float>(1 << (7 - t - 4 * half));
                int dd[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = 32 * w + t + 4 * half + 8 * i;
                    const float v = is_q ? sp[h][j] : coef * sq[h][j];
                    int d4[4];
                    digits4(__float2int_rn(v * fac / sig), d4);
                    dd[i] = d4[dig];
                }
                b[half] = pack4(dd[0], dd[1], dd[2], dd[3]);
            }
        }
        frag[e] = make_uint2(b[0], b[1]);
    }
}

// Bytes of one block's side record of a double-quantized NSN cache: fp16
// offset, step and norm step, 4-bit codes of the D block means and of the 128
// token norms, padded to a multiple of 16 bytes.
__host__ __device__ constexpr int dq_rec_bytes(int D) { return (8 + D / 2 + 64 + 15) / 16 * 16; }

// Shared-memory plan of the split kernel.  NSN: caches written by the NSN
// front end (no QJL), whose stages also carry the fp16 block means of keys
// and values (one D-vector per 128 tokens).  DQ (with NSN): the caches hold
// fp16 ||w|| per token and one side record per 128 tokens instead; the stage
// carries them as stored, and each sub-chunk expands them into fp32 norms
// (n1, ||w||) per token and fp32 block means in the expansion area.
template <int D, int B, bool QJL, int G, bool NSN = false, bool DQ = false>
struct MmaSmem {
    static constexpr int M = D;
    static constexpr int TC = DTile<D>::TC;
    static constexpr int NTK = HeadCfg<G>::NTK;
    static constexpr int RT = HeadCfg<G>::RT;
    static constexpr int GP = HeadCfg<G>::GP;
    static constexpr int KS = (PlaneCoefs<B>::PV + (QJL ? 1 : 0)) * (D / 32);
    // staging of one sub-chunk
    static constexpr int kKc = TC * B * D / 8;             // key codes (token layout)
    static constexpr int kKq = QJL ? TC * M / 8 : 0;       // key sign bits
    static constexpr int kKn = DQ ? TC * 2 : TC * 4;       // key norms
    static constexpr int kVc = (TC / 32) * B * D * 4;      // value codes (block-32)
    static constexpr int kVq = QJL ? (TC / 32) * M * 4 : 0;
    static constexpr int kVn = kKn;
    static constexpr int kNblk = (TC + 127) / 128;
    static constexpr int kKm = NSN ? kNblk * (DQ ? dq_rec_bytes(D) : D * 2) : 0;  // key block means
    static constexpr int kVm = kKm;                                                // value block means
    static constexpr int kStage = kKc + kKq + kKn + kVc + kVq + kVn + kKm + kVm;
    static constexpr int kXp = DQ ? 2 * TC * 8 + 2 * kNblk * D * 4 : 0;           // DQ expansion area
    static constexpr int kFrag = KS * NTK * 32 * 8;        // query fragments
    static constexpr int kLog = GP * TC * 4;               // logits of the sub-chunk
    static constexpr int kWfrag = (TC / 32) * RT * 32 * 16;  // weight digits, per kind
    static constexpr int kMisc = NSN ? 1536 : 1024;
    static constexpr int kBytes = 2 * kStage + kFrag + kLog + 2 * kWfrag + kMisc + kXp;
    // query fragments held in registers (at G <= 2 under the same K-step bound
    // as with two n-tiles: more live fragments cost a resident CTA per SM)
    static constexpr bool kQfReg = KS * (NTK == 1 ? 2 : NTK) <= 24;
};

template <int D, int B, bool QJL, int G, bool NSN = false, bool DQ = false>
__global__ void __launch_bounds__(kThreads) decode_mma_kernel(const __grid_constant__ DecodeArgs a) {
    static_assert(!(NSN && QJL), "NSN caches carry no QJL sketch");
    static_assert(!DQ || NSN, "double-quantized side data belong to NSN caches");
    using L = MmaSmem<D, B, QJL, G, NSN, DQ>;
    constexpr int RB = dq_rec_bytes(D);
    using HC = HeadCfg<G>;
    constexpr int M = D, TC = L::TC, NTK = L::NTK, RT = L::RT, KS = L::KS, GP = L::GP, CPL = HC::CPL;
    constexpr int KWT = B * D / 32;           // code words per token (key layout)
    constexpr int PV = PlaneCoefs<B>::PV;     // code planes incl. the parity plane (B = 3)
    constexpr int KWV = PV * D / 32;          // code-plane words per token, the parity plane included
    constexpr int QWT = QJL ? M / 32 : 0;     // sign words per token
    constexpr int NTV = D / 32;               // value n-tiles per warp (D/4 coordinates / 8)
    constexpr int NPV = PV + (QJL ? 1 : 0);
    constexpr bool QF_REG = L::kQfReg;
    constexpr int HH = (G == 8) ? 2 : 1;      // query heads per lane in the logit epilogue
    extern __shared__ __align__(128) uint8_t smem[];
    uint2* sfrag = reinterpret_cast<uint2*>(smem + 2 * L::kStage);
    float* slog = reinterpret_cast<float*>(smem + 2 * L::kStage + L::kFrag);  // [GP][TC]
    uint32_t* swc = reinterpret_cast<uint32_t*>(smem + 2 * L::kStage + L::kFrag + L::kLog);  // code-weight digits
    uint32_t* swq = swc + L::kWfrag / 4;                                                       // QJL-weight digits
    uint8_t* misc = smem + 2 * L::kStage + L::kFrag + L::kLog + 2 * L::kWfrag;
    uint64_t* bar = reinterpret_cast<uint64_t*>(misc);      // [2]
    float* sred = reinterpret_cast<float*>(misc + 16);      // 96 floats: [4 warps][GP][3] or [4 warps][16]
    float* shead = sred + 96;                                // [GP][8]: item sums (5..7)
    float* sstat = shead + GP * 8;                           // [GP][8]: -, alpha, sig_w/128, sig_wq/128
    float* sqo = sstat + GP * 8;                             // NSN: [GP][2] scale/sqrt(d) <q, o_k> per block
    float* sbeta = sqo + GP * 2;                             // NSN: [4 warps][GP][2] sums of e ||x||/sqrt(d)
    // DQ: per sub-chunk, (n1, ||w||) per token and the block means, in fp32
    float2* xkn = reinterpret_cast<float2*>(misc + L::kMisc);
    float2* xvn = xkn + (DQ ? L::TC : 0);
    float* xkm = reinterpret_cast<float*>(xvn + (DQ ? L::TC : 0));
    float* xvm = xkm + (DQ ? L::kNblk * D : 0);
    const float inv_sqrt_d = rsqrtf(static_cast<float>(D));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const uint32_t msk_lo = kLowBits << t, msk_hi = kLowBits << (t + 4);
    const float kappa = kSqrtHalfPi / M;
    const PlaneCoefs<B> pc = plane_coefs<B>(a.centroid);

    for (int e = tid; e < 2 * L::kWfrag / 4; e += kThreads) swc[e] = 0u;  // padding rows stay zero
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    uint32_t phase[2] = {0u, 0u};
    bool alive = true;
    const int64_t items = static_cast<int64_t>(a.batch) * a.hkv * a.nsplit_run;

    for (int64_t item = blockIdx.x; item < items && alive; item += gridDim.x) {
        const int split = static_cast<int>(item % a.nsplit_run);
        const int64_t stream = item / a.nsplit_run;
        const int hk = static_cast<int>(stream % a.hkv), bi = static_cast<int>(stream / a.hkv);
        const int64_t T = min(static_cast<int64_t>(max(a.seq_len[bi], 0)), a.max_T);
        const int64_t t0 = static_cast<int64_t>(split) * a.chunk;
        const int64_t t1e = min(t0 + a.chunk, a.max_T);
        const int64_t t1 = min(t1e, T);
        const int64_t qh0 = static_cast<int64_t>(bi) * a.hq + static_cast<int64_t>(hk) * G;
        const uint8_t* kc = reinterpret_cast<const uint8_t*>(a.kcodes) + stream * a.kcap * (B * D / 8);
        const uint8_t* kq = QJL ? reinterpret_cast<const uint8_t*>(a.kqjl) + stream * a.kcap * (M / 8) : nullptr;
        constexpr int NB = DQ ? 2 : 4;  // norm bytes per token
        const uint8_t* kn = reinterpret_cast<const uint8_t*>(a.knorms) + stream * a.kcap * NB;
        const uint8_t* vc = reinterpret_cast<const uint8_t*>(a.vcodes) + stream * (a.vcap / 32) * B * D * 4;
        const uint8_t* vq = QJL ? reinterpret_cast<const uint8_t*>(a.vqjl) + stream * (a.vcap / 32) * M * 4 : nullptr;
        const uint8_t* vn = reinterpret_cast<const uint8_t*>(a.vnorms) + stream * a.vcap * NB;
        // NSN: block means, [capacity / 128][D] fp16 per stream (DQ: side records of RB bytes)
        constexpr int MB = DQ ? RB : D * 2;  // bytes per block
        const uint8_t* km = NSN ? reinterpret_cast<const uint8_t*>(a.kmean) + stream * (a.kcap / 128) * MB : nullptr;
        const uint8_t* vm = NSN ? reinterpret_cast<const uint8_t*>(a.vmean) + stream * (a.vcap / 128) * MB : nullptr;

        // ---- item set-up (the previous item is done with shared memory) ----
        __syncthreads();
        {
            const uint2* gf = a.qfrag + stream * KS * NTK * 32;
            for (int e = tid; e < KS * NTK * 32; e += kThreads) sfrag[e] = gf[e];
        }
        // logit constants of this lane's heads t (and t + 4); with one key
        // n-tile (G <= 2) head t / 2:
        // l = n (k0 + k1 xc + n_gamma (k2 xq - k3)), scale / d folded in
        float hk0[HH], hk1[HH], hk2[HH], hk3[HH];
#pragma unroll
        for (int hh = 0; hh < HH; ++hh) {
            const int h = (NTK == 1) ? (t >> 1) : t + 4 * hh;
            hk0[hh] = hk1[hh] = hk2[hh] = hk3[hh] = 0.f;
            if (h < G) {
                const float* qs = a.qscal + (qh0 + h) * 4;
                const float f = a.scale / D;
                hk0[hh] = f * qs[0];
                hk1[hh] = f * qs[1];
                hk2[hh] = f * kappa * 2.f * qs[2];
                hk3[hh] = f * kappa * qs[3];
            }
        }
        // NSN: warp w holds the query of head w (and w + 4 when G = 8) in the
        // original domain, lane coordinates lane + 32 i, for <q, o_k> per block
        constexpr int QQ = (NSN && G == 8) ? 2 : 1;
        float qv[QQ][NSN ? D / 32 : 1];
        if constexpr (NSN) {
#pragma unroll
            for (int qq = 0; qq < QQ; ++qq) {
                const int h = warp + 4 * qq;
#pragma unroll
                for (int i = 0; i < D / 32; ++i)
                    qv[qq][i] = h < G ? load_elem_rt(a.q, a.qdtype, (qh0 + h) * D + lane + 32 * i) : 0.f;
            }
        }
        // running max per head (the same in every thread) and this thread's
        // partial sums of exp, code weights and QJL weights (rescaled with it)
        float mrun[GP], pe[GP], pw[GP], pq[GP];
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            mrun[h] = -INFINITY;
            pe[h] = pw[h] = pq[h] = 0.f;
        }
        const int nsub = static_cast<int>((t1e - t0 + TC - 1) / TC);
        // tokens of the sub-chunk that exist in the cache (rounded to whole blocks of 32)
        auto issue = [&](int sc) {
            const int64_t tb = t0 + static_cast<int64_t>(sc) * TC;
            const int64_t have = min(static_cast<int64_t>(TC), t1 - tb);
            if (have <= 0) return false;
            const int64_t nt = (have + 31) / 32 * 32;  // <= capacity - tb (capacity is a multiple of 32)
            uint8_t* st = smem + (sc & 1) * L::kStage;
            uint64_t* b = &bar[sc & 1];
            const int64_t nblk = NSN ? (nt + 127) / 128 : 0;  // block means of the sub-chunk
            const uint32_t bytes = static_cast<uint32_t>(nt * (B * D / 8 + (QJL ? M / 8 : 0) + NB) +
                                                         (nt / 32) * (B * D * 4 + (QJL ? M * 4 : 0)) + nt * NB +
                                                         2 * nblk * MB);
            mbar_arrive_expect_tx(b, bytes);
            bulk_load(st, kc + tb * (B * D / 8), static_cast<uint32_t>(nt * (B * D / 8)), b);
            if (QJL) bulk_load(st + L::kKc, kq + tb * (M / 8), static_cast<uint32_t>(nt * (M / 8)), b);
            bulk_load(st + L::kKc + L::kKq, kn + tb * NB, static_cast<uint32_t>(nt * NB), b);
            bulk_load(st + L::kKc + L::kKq + L::kKn, vc + (tb / 32) * B * D * 4,
                      static_cast<uint32_t>((nt / 32) * B * D * 4), b);
            if (QJL)
                bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc, vq + (tb / 32) * M * 4,
                          static_cast<uint32_t>((nt / 32) * M * 4), b);
            bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq, vn + tb * NB, static_cast<uint32_t>(nt * NB),
                      b);
            if (NSN) {
                const uint32_t mb = static_cast<uint32_t>(nblk * MB);
                bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq + L::kVn, km + (tb / 128) * MB, mb, b);
                bulk_load(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq + L::kVn + L::kKm, vm + (tb / 128) * MB,
                          mb, b);
            }
            return true;
        };
        bool armed0 = false, armed1 = false;
        if (tid == 0) {
            armed0 = issue(0);
            armed1 = nsub > 1 ? issue(1) : false;
        }
        __syncthreads();
        uint2 qf[QF_REG ? KS : 1][QF_REG ? NTK : 1];
        if (QF_REG) {
#pragma unroll
            for (int ks = 0; ks < (QF_REG ? KS : 1); ++ks)
#pragma unroll
                for (int nt = 0; nt < (QF_REG ? NTK : 1); ++nt) qf[ks][nt] = sfrag[(ks * NTK + nt) * 32 + lane];
        }

        // fp32 running value sums of this lane's (head, coordinate) pairs
        float accA[NTV][CPL], accB[NTV][CPL];
#pragma unroll
        for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
            for (int c = 0; c < CPL; ++c) accA[nt][c] = accB[nt][c] = 0.f;

        for (int sc = 0; sc < nsub; ++sc) {
            const int64_t tb = t0 + static_cast<int64_t>(sc) * TC;
            const int64_t have = min(static_cast<int64_t>(TC), t1 - tb);  // may be <= 0 (split past the context)
            const uint8_t* st = smem + (sc & 1) * L::kStage;
            // tokens of the sub-chunk inside the context, and inside the split (32-bit)
            const int nval = static_cast<int>(max(min(t1 - tb, static_cast<int64_t>(TC)), static_cast<int64_t>(0)));
            const int nval_e = static_cast<int>(max(min(t1e - tb, static_cast<int64_t>(TC)), static_cast<int64_t>(0)));
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
            const __half* sKm = reinterpret_cast<const __half*>(st + L::kKc + L::kKq + L::kKn + L::kVc + L::kVq + L::kVn);
            const __half* sVm = sKm + L::kKm / 2;
            if constexpr (DQ) {
                // Expand the sub-chunk's stored side data: n1 = q nstep and ||w|| per token,
                // o_hat = fp32(lo + step q) per block and channel (keys and values).
                const uint8_t* rk = reinterpret_cast<const uint8_t*>(sKm);
                const uint8_t* rv = rk + L::kKm;
                const __half* wk = reinterpret_cast<const __half*>(sKn);
                const __half* wv = reinterpret_cast<const __half*>(sVn);
                auto f16at = [](const uint8_t* p) { return __half2float(*reinterpret_cast<const __half*>(p)); };
                for (int tl = tid; tl < L::TC; tl += kThreads) {
                    const int bi = tl >> 7, tt = tl & 127;
                    const uint8_t* hk = rk + bi * RB;
                    const uint8_t* hv = rv + bi * RB;
                    const int qk = (hk[8 + D / 2 + tt / 2] >> ((tt & 1) * 4)) & 15;
                    const int qv2 = (hv[8 + D / 2 + tt / 2] >> ((tt & 1) * 4)) & 15;
                    xkn[tl] = make_float2(static_cast<float>(qk) * f16at(hk + 4), __half2float(wk[tl]));
                    xvn[tl] = make_float2(static_cast<float>(qv2) * f16at(hv + 4), __half2float(wv[tl]));
                }
                for (int e = tid; e < L::kNblk * D; e += kThreads) {
                    const int bi = e / D, j = e % D;
                    const uint8_t* hk = rk + bi * RB;
                    const uint8_t* hv = rv + bi * RB;
                    const int qk = (hk[8 + j / 2] >> ((j & 1) * 4)) & 15;
                    const int qv2 = (hv[8 + j / 2] >> ((j & 1) * 4)) & 15;
                    xkm[e] = fmaf(f16at(hk + 2), static_cast<float>(qk), f16at(hk));
                    xvm[e] = fmaf(f16at(hv + 2), static_cast<float>(qv2), f16at(hv));
                }
                __syncthreads();
            }
            // stored norms (||x|| or n1, then ||r|| or ||w||) and block means, as fp32
            auto knorm = [&](int tl) -> float2 { return DQ ? xkn[tl] : __half22float2(sKn[tl]); };
            auto vnorm = [&](int tl) -> float2 { return DQ ? xvn[tl] : __half22float2(sVn[tl]); };
            auto kmean = [&](int i) -> float { return DQ ? xkm[i] : __half2float(sKm[i]); };
            auto vmean = [&](int i) -> float { return DQ ? xvm[i] : __half2float(sVm[i]); };
            if constexpr (NSN) {
                // scale/sqrt(d) <q_h, o_k> for each 128-token block of the sub-chunk
                // (an unloaded block gives a value no valid token uses)
#pragma unroll
                for (int qq = 0; qq < QQ; ++qq)
#pragma unroll
                    for (int blk = 0; blk < (TC + 127) / 128; ++blk) {
                        float acc = 0.f;
#pragma unroll
                        for (int i = 0; i < D / 32; ++i)
                            acc = fmaf(qv[qq][i], kmean(blk * D + lane + 32 * i), acc);
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
                        const int h = warp + 4 * qq;
                        if (lane == 0 && h < GP) sqo[h * 2 + blk] = acc * a.scale * inv_sqrt_d;
                    }
                __syncthreads();
            }

            // ---------------- phase K: logits of the sub-chunk ----------------
            float lmax[HH];
#pragma unroll
            for (int hh = 0; hh < HH; ++hh) lmax[hh] = -INFINITY;
            for (int mt = warp; mt < TC / 16; mt += 4) {
                const int tl0 = mt * 16 + g, tl1 = tl0 + 8;
                int accc[2][NTK][4], accq[NTK][4];  // code K-steps alternate between two chains
                if (mt * 16 < nval) {
                    uint32_t w0[KS], w1[KS];
                    if constexpr (KWT % 4 == 0) {  // token records of 16-byte multiples
#pragma unroll
                        for (int q4 = 0; q4 < KWT / 4; ++q4) {
                            const uint4 x0 = reinterpret_cast<const uint4*>(sKc + tl0 * KWT)[q4];
                            const uint4 x1 = reinterpret_cast<const uint4*>(sKc + tl1 * KWT)[q4];
                            w0[4 * q4] = x0.x; w0[4 * q4 + 1] = x0.y; w0[4 * q4 + 2] = x0.z; w0[4 * q4 + 3] = x0.w;
                            w1[4 * q4] = x1.x; w1[4 * q4 + 1] = x1.y; w1[4 * q4 + 2] = x1.z; w1[4 * q4 + 3] = x1.w;
                        }
                    } else {  // 8-byte multiples (d = 64 with 1 or 3 bits)
#pragma unroll
                        for (int q2 = 0; q2 < KWT / 2; ++q2) {
                            const uint2 x0 = reinterpret_cast<const uint2*>(sKc + tl0 * KWT)[q2];
                            const uint2 x1 = reinterpret_cast<const uint2*>(sKc + tl1 * KWT)[q2];
                            w0[2 * q2] = x0.x; w0[2 * q2 + 1] = x0.y;
                            w1[2 * q2] = x1.x; w1[2 * q2 + 1] = x1.y;
                        }
                    }
                    if constexpr (PV > B) {
                        // the parity plane: bit0 ^ bit1 ^ bit2 of every coordinate
#pragma unroll
                        for (int w = 0; w < D / 32; ++w) {
                            w0[KWT + w] = w0[w] ^ w0[D / 32 + w] ^ w0[2 * (D / 32) + w];
                            w1[KWT + w] = w1[w] ^ w1[D / 32 + w] ^ w1[2 * (D / 32) + w];
                        }
                    }
                    if (QJL) {
#pragma unroll
                        for (int k = 0; k < QWT; k += 2) {
                            const uint2 x0 = reinterpret_cast<const uint2*>(sKq + tl0 * QWT)[k / 2];
                            const uint2 x1 = reinterpret_cast<const uint2*>(sKq + tl1 * QWT)[k / 2];
                            w0[KWV + k] = x0.x; w0[KWV + k + 1] = x0.y;
                            w1[KWV + k] = x1.x; w1[KWV + k + 1] = x1.y;
                        }
                    }
                    // code and QJL K-steps interleaved: 2 NTK independent accumulators
#pragma unroll
                    for (int i = 0; i < KWV || i < QWT; ++i) {
#pragma unroll
                        for (int kind = 0; kind < 2; ++kind) {
                            if (kind == 0 ? (i >= KWV) : (i >= QWT)) continue;
                            const int ks = kind == 0 ? i : KWV + i;
                            const uint4 af = make_uint4(w0[ks] & msk_lo, w1[ks] & msk_lo, w0[ks] & msk_hi,
                                                        w1[ks] & msk_hi);
#pragma unroll
                            for (int nt = 0; nt < NTK; ++nt) {
                                const uint2 bq = QF_REG ? qf[QF_REG ? ks : 0][QF_REG ? nt : 0]
                                                        : sfrag[(ks * NTK + nt) * 32 + lane];
                                if (kind == 0) {
                                    if (i < 2) mma_u8s8_qz(accc[i & 1][nt], af, bq);
                                    else mma_u8s8_q(accc[i & 1][nt], af, bq);
                                } else {
                                    if (i == 0) mma_u8s8_qz(accq[nt], af, bq);
                                    else mma_u8s8_q(accq[nt], af, bq);
                                }
                            }
                        }
                    }
                    if (KWV < 2) {
#pragma unroll
                        for (int nt = 0; nt < NTK; ++nt)
#pragma unroll
                            for (int r = 0; r < 4; ++r) accc[1][nt][r] = 0;
                    }
                } else {
#pragma unroll
                    for (int nt = 0; nt < NTK; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) accc[0][nt][r] = accc[1][nt][r] = accq[nt][r] = 0;
                }
                // epilogue: thread t owns head t (and t + 4 when G = 8); its
                // columns hold the four digits of the head.  With one key
                // n-tile (G <= 2) lanes t and t ^ 1 hold digits 0, 1 and 2, 3 of
                // head t / 2: one exchange completes both, and the even lane
                // keeps the logit.
                const bool own = (NTK > 1) || ((t & 1) == 0);
#pragma unroll
                for (int hh = 0; hh < HH; ++hh) {
                    const int h = (NTK == 1) ? (t >> 1) : t + 4 * hh;
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int tl = rr ? tl1 : tl0;
                        float l;
                        {
                            float xc, xq = 0.f;
                            if constexpr (NTK == 1) {
                                const int mine = (accc[0][0][2 * rr] + accc[1][0][2 * rr]) * 128 + accc[0][0][2 * rr + 1] +
                                                 accc[1][0][2 * rr + 1];
                                const int other = __shfl_xor_sync(0xFFFFFFFFu, mine, 1);
                                xc = fmaf(static_cast<float>((t & 1) ? other : mine), 16384.f,
                                          static_cast<float>((t & 1) ? mine : other));
                                if (QJL) {
                                    const int mq = accq[0][2 * rr] * 128 + accq[0][2 * rr + 1];
                                    const int oq = __shfl_xor_sync(0xFFFFFFFFu, mq, 1);
                                    xq = fmaf(static_cast<float>((t & 1) ? oq : mq), 16384.f,
                                              static_cast<float>((t & 1) ? mq : oq));
                                }
                            } else {
                                const int n0 = 2 * hh, n1 = 2 * hh + 1;
                                xc = fmaf(static_cast<float>((accc[0][n0][2 * rr] + accc[1][n0][2 * rr]) * 128 +
                                                             accc[0][n0][2 * rr + 1] + accc[1][n0][2 * rr + 1]),
                                          16384.f,
                                          static_cast<float>((accc[0][n1][2 * rr] + accc[1][n1][2 * rr]) * 128 +
                                                             accc[0][n1][2 * rr + 1] + accc[1][n1][2 * rr + 1]));
                                if (QJL)
                                    xq = fmaf(static_cast<float>(accq[n0][2 * rr] * 128 + accq[n0][2 * rr + 1]), 16384.f,
                                              static_cast<float>(accq[n1][2 * rr] * 128 + accq[n1][2 * rr + 1]));
                            }
                            const float2 nk = knorm(tl);
                            float inner = fmaf(hk1[hh], xc, hk0[hh]);
                            if (QJL) inner = fmaf(nk.y, fmaf(hk2[hh], xq, -hk3[hh]), inner);
                            // NSN: l = scale ||x||/sqrt(d) (||w||/d <q', c> + <q, o>)
                            const float lt = NSN ? nk.x * fmaf(nk.y * inv_sqrt_d, inner, sqo[h * 2 + (tl >> 7)])
                                                 : nk.x * inner;
                            l = (own && h < G && tl < nval) ? lt : -INFINITY;
                            lmax[hh] = fmaxf(lmax[hh], l);
                        }
                        if (own && h < GP) slog[h * TC + tl] = l;
                        if (own && a.logits != nullptr && h < G && tl < nval_e)
                            a.logits[(qh0 + h) * a.logits_ld + tb + tl] = l;
                    }
                }
            }
            // Bounds for the weight digits: per head the max logit of the
            // sub-chunk, and the max value norm n (and n gamma); the product
            // bounds the largest weight.
            {
                float nmx = 0.f, ngx = 0.f;
                for (int tl = tid; tl < TC; tl += kThreads) {
                    if (tl < nval) {
                        const float2 nv = vnorm(tl);
                        nmx = fmaxf(nmx, NSN ? nv.x * nv.y * inv_sqrt_d : nv.x);
                        ngx = fmaxf(ngx, nv.x * nv.y);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    nmx = fmaxf(nmx, __shfl_xor_sync(0xFFFFFFFFu, nmx, o));
                    ngx = fmaxf(ngx, __shfl_xor_sync(0xFFFFFFFFu, ngx, o));
                }
#pragma unroll
                for (int hh = 0; hh < HH; ++hh)
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) lmax[hh] = fmaxf(lmax[hh], __shfl_xor_sync(0xFFFFFFFFu, lmax[hh], o));
                if (g == 0) {
#pragma unroll
                    for (int hh = 0; hh < HH; ++hh)
                        if (NTK == 1) sred[warp * 16 + ((t & 1) ? 2 + (t >> 1) : (t >> 1))] = lmax[hh];  // odd lanes: -inf
                        else if (t + 4 * hh < GP) sred[warp * 16 + t + 4 * hh] = lmax[hh];
                }
                if (lane == 0) {
                    sred[warp * 16 + 8] = nmx;
                    sred[warp * 16 + 9] = ngx;
                }
            }
            __syncthreads();
            // Softmax statistics of the sub-chunk, computed alike by every
            // thread: new running max, rescale factor, digit scales (weight w
            // is the integer w 2^(7-s) inv < kWCap; a digit sum S of the value
            // MMA stands for S sig / 128 with sig = 1 / inv).
            float mnew[GP], invw[GP], invq[GP];
            {
                // lane h < GP of every warp works out head h; the others take
                // the values by shuffle
                float nmax = 0.f, ngmax = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    nmax = fmaxf(nmax, sred[w * 16 + 8]);
                    ngmax = fmaxf(ngmax, sred[w * 16 + 9]);
                }
                const int hl = lane < GP ? lane : 0;
                float msc = -INFINITY;
#pragma unroll
                for (int w = 0; w < 4; ++w) msc = fmaxf(msc, sred[w * 16 + hl]);
                float mold = mrun[0];
#pragma unroll
                for (int h = 1; h < GP; ++h) mold = (hl == h) ? mrun[h] : mold;
                const float mn = fmaxf(mold, msc);
                const float al = (mn == -INFINITY) ? 1.f : __expf(mold - mn);
                const float top = (msc == -INFINITY) ? 0.f : __expf(msc - mn);
                const float wb = top * nmax, qb = top * ngmax;
                const float iw = wb > 0.f ? __fdividef(kWCap / 128.f, wb) : 0.f;
                const float iq = qb > 0.f ? __fdividef(kWCap / 128.f, qb) : 0.f;
                if (warp == 0 && lane < GP) {
                    sstat[lane * 8 + 1] = al;
                    sstat[lane * 8 + 2] = iw > 0.f ? __fdividef(1.f / 128.f, iw) : 0.f;  // sig / 128
                    sstat[lane * 8 + 3] = iq > 0.f ? __fdividef(1.f / 128.f, iq) : 0.f;
                }
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    mnew[h] = __shfl_sync(0xFFFFFFFFu, mn, h);
                    invw[h] = __shfl_sync(0xFFFFFFFFu, iw, h);
                    invq[h] = __shfl_sync(0xFFFFFFFFu, iq, h);
                    const float alpha = __shfl_sync(0xFFFFFFFFu, al, h);
                    mrun[h] = mnew[h];
                    pe[h] *= alpha;
                    pw[h] *= alpha;
                    pq[h] *= alpha;
                }
            }
            // pass 2: weight digits into A-fragment bytes; partial sums.
            // Token u of block bb is K index 4(u&7) + (u>>3) (u&7 < 4) or
            // 16 + 4((u&7)-4) + (u>>3): lane 4(r&7) + (u&3), register
            // (r>>3) + 2((u&7)>>2), byte u>>3 of row r's fragment.
            for (int tl = tid; tl < TC; tl += kThreads) {
                const bool valid = tl < nval;
                const float2 nv = valid ? vnorm(tl) : make_float2(0.f, 0.f);
                const int u = tl & 31, bb = tl >> 5, s = u & 7;
                const float fac = static_cast<float>(1 << (7 - s));
                uint8_t* bc = reinterpret_cast<uint8_t*>(swc) + (u >> 3);
                uint8_t* bq = reinterpret_cast<uint8_t*>(swq) + (u >> 3);
                // NSN: the code weight is e ||x|| ||w|| / sqrt(d); the block mean
                // enters with e ||x|| / sqrt(d), summed per head over the block
                const float nwc = NSN ? nv.x * nv.y * inv_sqrt_d : nv.x;
                float eb[NSN ? GP : 1];
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    uint32_t xc, xq = 0u;
                    {
                        const float ex = __expf(slog[h * TC + tl] - mnew[h]);
                        const float e = (valid && h < G) ? ex : 0.f;
                        if (NSN) eb[NSN ? h : 0] = e * nv.x * inv_sqrt_d;
                        const float wc = e * nwc;
                        const float wq = wc * nv.y;
                        pe[h] += e;
                        pw[h] += wc;
                        pq[h] += wq;
                        xc = __float2uint_rn(wc * (fac * invw[h]));
                        if (QJL) xq = __float2uint_rn(wq * (fac * invq[h]));
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // row r of the weight operand: G <= 4: r = h + 4k; G = 8: r = h + 8k
                        const int r = (G <= 4) ? h + 4 * k : h + 8 * k;
                        const int rt = r >> 4, rl = r & 15;
                        const int off =
                            ((((bb * RT + rt) * 32 + 4 * (rl & 7) + (s & 3)) * 4 + (rl >> 3) + 2 * (s >> 2)) << 2);
                        bc[off] = static_cast<uint8_t>(xc >> (8 * k));
                        if (QJL) bq[off] = static_cast<uint8_t>(xq >> (8 * k));
                    }
                }
                if constexpr (NSN) {
                    // every token of this pass is in block tl >> 7 (tl = tid + 128 i)
#pragma unroll
                    for (int h = 0; h < GP; ++h) {
                        float v = eb[h];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                        if (lane == 0) sbeta[(warp * GP + h) * 2 + (tl >> 7)] = v;
                    }
                }
            }
            __syncthreads();

            // ---------------- phase V: value sums of the sub-chunk ----------------
            // Lane (g, t) of warp w reads the words of coordinates
            // w D/4 + NTV g + nt (nt < NTV) in one load: n-tile nt, column n is
            // coordinate w D/4 + NTV n + nt.
            {
                int accv[NPV][NTV][RT][4];
                const int nblk = nval > 0 ? (nval + 31) / 32 : 0;
                const int cbase = warp * (D / 4) + NTV * g;
                auto vblock = [&](int bb, bool first) {
                    uint4 aw[RT], aq[RT];
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt) {
                        aw[rt] = reinterpret_cast<const uint4*>(swc)[(bb * RT + rt) * 32 + lane];
                        if (QJL) aq[rt] = reinterpret_cast<const uint4*>(swq)[(bb * RT + rt) * 32 + lane];
                    }
                    uint32_t wr[3][NTV];  // real planes' words, for the parity plane (B = 3)
#pragma unroll
                    for (int p = 0; p < NPV; ++p) {
                        uint32_t wv[NTV];
                        if (PV > B && p == B) {
#pragma unroll
                            for (int nt = 0; nt < NTV; ++nt) wv[nt] = wr[0][nt] ^ wr[1][nt] ^ wr[2][nt];
                        } else {
                            const uint32_t* src = (p < B) ? sVc + (bb * B + p) * D + cbase : sVq + bb * M + cbase;
                            if (NTV % 4 == 0) {
#pragma unroll
                                for (int q4 = 0; q4 < NTV / 4; ++q4) {
                                    const uint4 x = reinterpret_cast<const uint4*>(src)[q4];
                                    wv[4 * q4] = x.x; wv[4 * q4 + 1] = x.y; wv[4 * q4 + 2] = x.z;
                                    wv[4 * q4 + 3] = x.w;
                                }
                            } else {
#pragma unroll
                                for (int q2 = 0; q2 < NTV / 2; ++q2) {
                                    const uint2 x = reinterpret_cast<const uint2*>(src)[q2];
                                    wv[2 * q2] = x.x; wv[2 * q2 + 1] = x.y;
                                }
                            }
                            if (PV > B && p < B) {
#pragma unroll
                                for (int nt = 0; nt < NTV; ++nt) wr[p < 3 ? p : 0][nt] = wv[nt];
                            }
                        }
#pragma unroll
                        for (int nt = 0; nt < NTV; ++nt) {
                            const uint2 bv = make_uint2(wv[nt] & msk_lo, wv[nt] & msk_hi);
#pragma unroll
                            for (int rt = 0; rt < RT; ++rt) {
                                const uint4 af = (p < PV) ? aw[rt] : aq[(QJL ? rt : 0)];
                                if (first) mma_u8u8_qz(accv[p][nt][rt], af, bv);
                                else mma_u8u8_q(accv[p][nt][rt], af, bv);
                            }
                        }
                    }
                };
                if (nblk > 0) {
                    vblock(0, true);
                    for (int bb = 1; bb < nblk; ++bb) vblock(bb, false);
                } else {
#pragma unroll
                    for (int p = 0; p < NPV; ++p)
#pragma unroll
                        for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
                            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                                for (int r = 0; r < 4; ++r) accv[p][nt][rt][r] = 0;
                }
                // Merge into the fp32 running sums (rescaled by alpha).  Digit k
                // of head h sits in row h + 4k (G <= 4): lane g < 4 holds digits
                // 0, 2 of head g and lane + 16 digits 1, 3; lane g < 4 completes
                // column 2t, lane g + 4 column 2t + 1, swapping the other two.
                // With G = 8 (rows h + 8k, two row tiles) every lane holds all
                // digits of head g, columns 2t and 2t + 1.  Each digit sum is
                // non-negative and below 2^24.
                const int head = (G <= 4) ? (g & 3) : g;
                const bool hi = g >= 4;
                const float* ss = sstat + (head < G ? head : 0) * 8;
                const float alpha = ss[1];
                const float sgw = ss[2];
                const float sgq = ss[3];
#pragma unroll
                for (int nt = 0; nt < NTV; ++nt) {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        float vals[NPV];
#pragma unroll
                        for (int p = 0; p < NPV; ++p) {
                            uint32_t d0, d1, d2, d3;
                            if (G <= 4) {
                                const int* x = accv[p][nt][0];
                                const int s1 = __shfl_xor_sync(0xFFFFFFFFu, hi ? x[0] : x[1], 16);
                                const int s3 = __shfl_xor_sync(0xFFFFFFFFu, hi ? x[2] : x[3], 16);
                                d0 = static_cast<uint32_t>(hi ? s1 : x[0]);
                                d1 = static_cast<uint32_t>(hi ? x[1] : s1);
                                d2 = static_cast<uint32_t>(hi ? s3 : x[2]);
                                d3 = static_cast<uint32_t>(hi ? x[3] : s3);
                            } else {
                                d0 = static_cast<uint32_t>(accv[p][nt][0][c]);
                                d1 = static_cast<uint32_t>(accv[p][nt][0][2 + c]);
                                d2 = static_cast<uint32_t>(accv[p][nt][RT - 1][c]);
                                d3 = static_cast<uint32_t>(accv[p][nt][RT - 1][2 + c]);
                            }
                            vals[p] = fmaf(static_cast<float>(d3), 16777216.f,
                                           fmaf(static_cast<float>(d2), 65536.f, static_cast<float>(d1 * 256u + d0)));
                        }
                        if (head < G) {
                            float code = pc.coef[0] * vals[0];
#pragma unroll
                            for (int v = 1; v < PV; ++v) code = fmaf(pc.coef[v], vals[v], code);
                            accA[nt][c] = fmaf(accA[nt][c], alpha, sgw * code);
                            if (QJL) accB[nt][c] = fmaf(accB[nt][c], alpha, sgq * 2.f * vals[NPV - 1]);
                            if (NSN) {
                                // O += sum_blk beta_blk o_v,blk on this lane's (head, coordinate),
                                // in the original (unrotated) coordinates; unloaded blocks are skipped
                                const int col = (G <= 4) ? 2 * t + (g >= 4 ? 1 : 0) : 2 * t + c;
                                const int coord = warp * (D / 4) + NTV * col + nt;
                                float add = 0.f;
#pragma unroll
                                for (int blk = 0; blk < (TC + 127) / 128; ++blk) {
                                    if (nval > blk * 128) {
                                        float bsum = 0.f;
#pragma unroll
                                        for (int w = 0; w < 4; ++w) bsum += sbeta[(w * GP + head) * 2 + blk];
                                        add = fmaf(bsum, vmean(blk * D + coord), add);
                                    }
                                }
                                accB[nt][c] = fmaf(accB[nt][c], alpha, add);
                            }
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
        if (!alive) {
            if (tid == 0) {
                // loads in flight are waited for before exit (only when a wait gave up)
                if (armed0) mbar_wait(&bar[0], phase[0], a.status);
                if (armed1) mbar_wait(&bar[1], phase[1], a.status);
            }
            break;
        }

        // ---------------- partials: {M, L, A[D], B[M]} per query head ----------------
        // CTA-wide sums of this item's exp and weights (shead[h*8 + 5..7]).
        {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    pe[h] += __shfl_xor_sync(0xFFFFFFFFu, pe[h], o);
                    pw[h] += __shfl_xor_sync(0xFFFFFFFFu, pw[h], o);
                    pq[h] += __shfl_xor_sync(0xFFFFFFFFu, pq[h], o);
                }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    sred[(warp * GP + h) * 3 + 0] = pe[h];
                    sred[(warp * GP + h) * 3 + 1] = pw[h];
                    sred[(warp * GP + h) * 3 + 2] = pq[h];
                }
            __syncthreads();
            if (tid < GP) {
                float te = 0.f, tw = 0.f, twq = 0.f;
                for (int w = 0; w < 4; ++w) {
                    te += sred[(w * GP + tid) * 3 + 0];
                    tw += sred[(w * GP + tid) * 3 + 1];
                    twq += sred[(w * GP + tid) * 3 + 2];
                }
                shead[tid * 8 + 5] = te;
                shead[tid * 8 + 6] = tw;
                shead[tid * 8 + 7] = twq;
            }
            __syncthreads();
        }
        constexpr int PART = 2 + D + M;
        {
            const int head = (G <= 4) ? (g & 3) : g;
            if (head < G) {
                float* pp = a.part + ((qh0 + head) * a.nsplit + split) * PART;
                const float* hs = shead + head * 8;
                const float c0 = pc.cst;
#pragma unroll
                for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const int col = (G <= 4) ? 2 * t + (g >= 4 ? 1 : 0) : 2 * t + c;
                        const int coord = warp * (D / 4) + NTV * col + nt;
                        pp[2 + coord] = c0 * hs[6] + accA[nt][c];
                        if (QJL) pp[2 + D + coord] = accB[nt][c] - hs[7];
                        if (NSN) pp[2 + D + coord] = accB[nt][c];
                    }
            }
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                if (tid == h && h < G) {
                    float* pp = a.part + ((qh0 + h) * a.nsplit + split) * PART;
                    pp[0] = mrun[h];
                    pp[1] = shead[h * 8 + 5];
                }
            }
        }
    }
}

template <int D, int B, bool QJL, int G, bool NSN = false, bool DQ = false>
int ctas_per_sm_g() {
    using L = MmaSmem<D, B, QJL, G, NSN, DQ>;
    auto kern = decode_mma_kernel<D, B, QJL, G, NSN, DQ>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess) return 1;
    int n = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, L::kBytes) != cudaSuccess || n < 1) n = 1;
    return n;
}

template <int D, int B, bool QJL>
int ctas_per_sm_d(int G) {
    switch (G) {
        case 1: return ctas_per_sm_g<D, B, QJL, 1>();
        case 2: return ctas_per_sm_g<D, B, QJL, 2>();
        case 4: return ctas_per_sm_g<D, B, QJL, 4>();
        default: return ctas_per_sm_g<D, B, QJL, 8>();
    }
}

template <int D, int B, bool QJL, int G>
cudaError_t launch_mma_g(const DecodeArgs& a, int grid, cudaStream_t s) {
    const int groups = a.batch * a.hkv;
    switch (a.qdtype) {
        case 0: qfrag_kernel<D, B, QJL, G, 0><<<groups, kThreads, 0, s>>>(a); break;
        case 1: qfrag_kernel<D, B, QJL, G, 1><<<groups, kThreads, 0, s>>>(a); break;
        default: qfrag_kernel<D, B, QJL, G, 2><<<groups, kThreads, 0, s>>>(a); break;
    }
    const int64_t items = static_cast<int64_t>(a.batch) * a.hkv * a.nsplit_run;
    if constexpr (!QJL) {
        if (a.nsn) {
            // NSN caches (fp16 or double-quantized side data): the same split
            // plan, on the variant's own persistent grid
            auto run = [&](auto dq) -> cudaError_t {
                constexpr bool DQ = decltype(dq)::value;
                using LN = MmaSmem<D, B, false, G, true, DQ>;
                auto kn = decode_mma_kernel<D, B, false, G, true, DQ>;
                cudaError_t e = cudaFuncSetAttribute(kn, cudaFuncAttributeMaxDynamicSharedMemorySize, LN::kBytes);
                if (e != cudaSuccess) return e;
                int sms = 148, dev = 0;
                cudaGetDevice(&dev);
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
                const int64_t gn = static_cast<int64_t>(ctas_per_sm_g<D, B, false, G, true, DQ>()) * sms;
                const int64_t n = items < gn ? items : gn;
                if (n <= 0) return cudaSuccess;
                kn<<<static_cast<unsigned>(n), kThreads, LN::kBytes, s>>>(a);
                return cudaGetLastError();
            };
            return a.nsn_dq ? run(std::true_type()) : run(std::false_type());
        }
    }
    using L = MmaSmem<D, B, QJL, G>;
    auto kern = decode_mma_kernel<D, B, QJL, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    const int64_t n = items < grid ? items : grid;
    if (n <= 0) return cudaSuccess;
    kern<<<static_cast<unsigned>(n), kThreads, L::kBytes, s>>>(a);
    return cudaGetLastError();
}

template <int D, int B, bool QJL>
cudaError_t launch_mma_d(const DecodeArgs& a, int grid, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_mma_g<D, B, QJL, 1>(a, grid, s);
        case 2: return launch_mma_g<D, B, QJL, 2>(a, grid, s);
        case 4: return launch_mma_g<D, B, QJL, 4>(a, grid, s);
        default: return launch_mma_g<D, B, QJL, 8>(a, grid, s);
    }
}

}  // namespace

#define KVQ_MMA_CASES(FN, ...)                                              \
    switch (h->d * 16 + h->b * 4 + (qjl ? 1 : 0)) {                         \
        case 64 * 16 + 4: return FN<64, 1, false>(__VA_ARGS__);             \
        case 64 * 16 + 5: return FN<64, 1, true>(__VA_ARGS__);              \
        case 64 * 16 + 8: return FN<64, 2, false>(__VA_ARGS__);             \
        case 64 * 16 + 9: return FN<64, 2, true>(__VA_ARGS__);              \
        case 128 * 16 + 4: return FN<128, 1, false>(__VA_ARGS__);           \
        case 128 * 16 + 5: return FN<128, 1, true>(__VA_ARGS__);            \
        case 128 * 16 + 8: return FN<128, 2, false>(__VA_ARGS__);           \
        case 128 * 16 + 9: return FN<128, 2, true>(__VA_ARGS__);            \
        case 256 * 16 + 4: return FN<256, 1, false>(__VA_ARGS__);           \
        case 256 * 16 + 5: return FN<256, 1, true>(__VA_ARGS__);            \
        case 256 * 16 + 8: return FN<256, 2, false>(__VA_ARGS__);           \
        case 64 * 16 + 12: return FN<64, 3, false>(__VA_ARGS__);            \
        case 64 * 16 + 13: return FN<64, 3, true>(__VA_ARGS__);             \
        case 128 * 16 + 12: return FN<128, 3, false>(__VA_ARGS__);          \
        case 128 * 16 + 13: return FN<128, 3, true>(__VA_ARGS__);           \
        case 256 * 16 + 9: return FN<256, 2, true>(__VA_ARGS__);            \
        default: break;                                                     \
    }

namespace {
int ctas_per_sm(const kvq_ctx* h, int G) {
    const bool qjl = (h->flags & 1u) != 0;
    KVQ_MMA_CASES(ctas_per_sm_d, G)
    return 1;
}
}  // namespace

// Resident CTAs of the split kernel on the whole device: the persistent grid.
int decode_mma_grid(const kvq_ctx* h, int G) {
    const int gi = (G >= 1 && G <= 8) ? G : 8;
    if (h->mma_grid[gi] > 0) return h->mma_grid[gi];
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
    const int n = ctas_per_sm(h, G) * sms;
    const_cast<kvq_ctx*>(h)->mma_grid[gi] = n;
    return n;
}

// Query fragments + split kernel of the tensor-core path (decode_uses_mma).
cudaError_t launch_decode_mma(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s) {
    const bool qjl = (h->flags & 1u) != 0;
    const int grid = decode_mma_grid(h, a.G);
    KVQ_MMA_CASES(launch_mma_d, a, grid, s)
    return cudaErrorNotSupported;
}

size_t decode_mma_qfrag_bytes(const kvq_ctx* h, int G) {
    const int NTK = (G <= 2) ? 1 : (G <= 4) ? 2 : 4;
    const int PV = h->b == 3 ? 4 : h->b;  // code planes, the 3-bit parity plane included
    const int KS = (PV + ((h->flags & 1u) ? 1 : 0)) * (h->d / 32);
    return static_cast<size_t>(KS) * NTK * 32 * 8;
}

}  // namespace kvq
