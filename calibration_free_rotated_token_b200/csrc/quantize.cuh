// quantize.cuh -- the quantize kernel (and its NSN front-end variant).
//
// Method (TurboQuant blog, "Estagio 1" and "Estagio 2"; PolarQuant section 2;
// NSNQuant sections 1-2 for the front end), per vector x of dimension D:
//   n = ||x||, z = H (delta .* x) / n, code_j = #{k : z_j >= t_k},
//   r = z - c[code], gamma = ||r||, QJL bits = [S r >= 0], norms fp16.
//
// Design (sm_100a):
// * Persistent CTAs, one per SM, two warpgroups (256 threads).  128-vector
//   tiles stream through a ring of shared-memory stages with TMA (128-byte
//   swizzle, so that a thread reading "its" row is bank-conflict free); as
//   soon as a warpgroup has read a stage, its leader refills that stage with
//   the tile kStages ahead, so loads run that far ahead of the compute.
//   Tails past n are zero-filled by TMA and never stored.
// * One thread owns one vector (D <= 128) or one half of it (D = 256: the two
//   warpgroups cooperate on one tile and the top butterfly of the Hadamard
//   transform is taken at load time).  The FWHT runs entirely in registers:
//   no shuffles, no shared-memory round trips.
// * Codes are written as bit planes built in registers; the residual r is
//   rounded once to fp16 and stored into tensor memory (thread = TMEM lane =
//   MMA row), and one elected thread issues tcgen05 MMAs D(128 x m) = A S^T
//   with S (fp16, exact) resident in shared memory.  The epilogue reads its
//   own accumulator row back from TMEM and packs the sign bits.  The error of
//   (S r)_i is about 2e-4 ||r||, so a sign can differ from the exact one
//   outside a 1e-3 ||r|| band only through a 5-sigma error (~1e-11 per bit).
// * Every wait on an mbarrier is bounded; the outcome is agreed on by the
//   whole warpgroup (barrier reduction) so no thread is left at a barrier.
#pragma once

#include <cfloat>

#include "kvq_internal.h"
#include "sm100.cuh"

namespace kvq {

enum { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

template <int D, int B, bool QJL, int DT, bool NSN>
struct QCfg {
    static constexpr int kEsz = (DT == DT_F32) ? 4 : 2;
    static constexpr int kBoxCols = 128 / kEsz;            // elements per 128-byte box row
    static constexpr int kBoxes = D * kEsz / 128;
    static constexpr int kBoxBytes = 128 * kTileRows;      // 16 KB
    static constexpr int kStageBytes = kBoxes * kBoxBytes;
    static constexpr bool kCoop = (D == 256);              // two threads per vector
    static constexpr int kNV = kCoop ? 128 : D;            // coordinates held per thread
    static constexpr int kSBytes = QJL ? D * D * 2 : 0;    // S, fp16, m = D rows
    static constexpr int kBudget = 200 * 1024;
    static constexpr int kStagesRaw = (kBudget - kSBytes) / kStageBytes;
    static constexpr int kStagesCap = kStagesRaw > 4 ? 4 : kStagesRaw;
    // Without cooperation each warpgroup owns the stages of its tiles (tile i
    // uses stage i % kStages and goes to warpgroup i % 2), so the count is even.
    static constexpr int kStages = kCoop ? kStagesCap : (kStagesCap & ~1);
    static constexpr int kThreads = 256;
    static constexpr int kTmemCols = !QJL ? 0 : (kCoop ? 512 : (4 * D < 32 ? 32 : 4 * D));
    static constexpr int kAuxBytes = NSN ? 8192 : 4096;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kSBytes + kAuxBytes;
    static_assert(kStages >= 1, "input tile does not fit in shared memory");
    static_assert(!(NSN && QJL), "NSN front end: no QJL");
    static_assert(!(NSN && kCoop), "NSN front end at D = 256: the tensor-core kernel");
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// Collect the sign bit of `x` as the new low bit of w (shifting w up by one).
__device__ __forceinline__ uint32_t push_sign(uint32_t w, float x) { return __funnelshift_l(f2u(x), w, 1); }

// Load this thread's row (D <= 128) from a swizzled stage as coordinate pairs
// v[k] = (x_2k, x_2k+1), applying the Rademacher signs when SIGN (XOR of the
// element sign bits).
template <int D, int DT, bool SIGN>
__device__ __forceinline__ void load_row(const uint8_t* sp, int r, float2 (&v)[D / 2], const uint32_t* psign) {
    constexpr int kEsz = DT == DT_F32 ? 4 : 2;
    constexpr int kEpc = 16 / kEsz;  // elements per 16-byte chunk
#pragma unroll
    for (int box = 0; box < D * kEsz / 128; ++box) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(sp + box * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            const int e0 = box * (128 / kEsz) + c * kEpc;
            if (DT == DT_F32) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int e = e0 + 2 * k;
                    uint32_t s0 = 0, s1 = 0;
                    if (SIGN) {
                        s0 = psign[e >> 1] << 16;
                        s1 = psign[e >> 1] & 0x80000000u;
                    }
                    v[e >> 1] = make_float2(u2f(w[2 * k] ^ (s0 & 0x80000000u)), u2f(w[2 * k + 1] ^ s1));
                }
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int pk = e0 / 2 + k;
                    const uint32_t wd = w[k] ^ (SIGN ? psign[pk] : 0u);
                    if (DT == DT_BF16) {
                        v[pk] = make_float2(u2f(wd << 16), u2f(wd & 0xFFFF0000u));
                    } else {
                        v[pk] = __half22float2(*reinterpret_cast<const __half2*>(&wd));
                    }
                }
            }
        }
    }
}

// D = 256, 16-bit input: half h of the rotated vector needs
// v_j = delta_j x_j + (-1)^h delta_{j+128} x_{j+128}, j < 128 (the top
// butterfly of the Sylvester transform), plus the full ||x||^2.
template <int DT>
__device__ __forceinline__ float load_row_coop(const uint8_t* sp, int r, int h, float2 (&v)[64],
                                               const uint32_t* psign) {
    float2 ss = make_float2(0.f, 0.f);
    const float2 sgn = h ? make_float2(-1.f, -1.f) : make_float2(1.f, 1.f);
#pragma unroll
    for (int box = 0; box < 2; ++box) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int off = r * 128 + ((c ^ (r & 7)) << 4);
            const uint4 qa = *reinterpret_cast<const uint4*>(sp + box * 16384 + off);
            const uint4 qb = *reinterpret_cast<const uint4*>(sp + (box + 2) * 16384 + off);
            const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
            const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int pk = box * 32 + c * 4 + k;  // pair index within the half
                const uint32_t xa = wa[k] ^ psign[pk];
                const uint32_t xb = wb[k] ^ psign[pk + 64];
                float2 a, b;
                if (DT == DT_BF16) {
                    a = make_float2(u2f(xa << 16), u2f(xa & 0xFFFF0000u));
                    b = make_float2(u2f(xb << 16), u2f(xb & 0xFFFF0000u));
                } else {
                    a = __half22float2(*reinterpret_cast<const __half2*>(&xa));
                    b = __half22float2(*reinterpret_cast<const __half2*>(&xb));
                }
                ss = __ffma2_rn(a, a, ss);
                ss = __ffma2_rn(b, b, ss);
                v[pk] = __ffma2_rn(sgn, b, a);
            }
        }
    }
    return ss.x + ss.y;
}

template <int NP>
__device__ __forceinline__ float sumsq(const float2 (&v)[NP]) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < NP; k += 2) {
        a = __ffma2_rn(v[k], v[k], a);
        b = __ffma2_rn(v[k + 1], v[k + 1], b);
    }
    a = __fadd2_rn(a, b);
    return a.x + a.y;
}

// In-register fast Walsh-Hadamard transform (Sylvester order, unnormalised)
// of 2*NP coordinates held as pairs: the stride-1 butterflies inside each
// pair, the others on whole pairs with packed fp32x2 adds.
template <int NP>
__device__ __forceinline__ void fwht(float2 (&v)[NP]) {
    const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
    for (int k = 0; k < NP; ++k) v[k] = make_float2(v[k].x + v[k].y, v[k].x - v[k].y);
#pragma unroll
    for (int hp = 1; hp < NP; hp <<= 1) {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            if ((k & hp) == 0) {
                const float2 a = v[k], b = v[k + hp];
                v[k] = __fadd2_rn(a, b);
                v[k + hp] = __ffma2_rn(b, m1, a);
            }
        }
    }
}

// Lloyd-Max cell of one coordinate z on the symmetric codebook, by sign and
// magnitude: the sign picks the half (the middle decision level is 0), and
// the magnitude |z| is compared with the positive decision levels
// tau_j = t[H-1+j] (binary search, H = 2^(B-1)); mu = c[H + idx] is the
// magnitude of the centroid.  g[p] = |z| - (level compared at search step p):
// its sign bit is the complement of magnitude-index bit p.  The levels and
// magnitudes sit in registers (MagTab), so every step is a compare and a
// register select: no branch and no indexed constant load.
template <int B>
struct MagTab {
    static constexpr int H = 1 << (B - 1);
    float tau[H];  // tau[0] unused
    float mu[H];
    __device__ __forceinline__ explicit MagTab(const QuantArgs& a) {
#pragma unroll
        for (int j = 0; j < H; ++j) {
            tau[j] = j > 0 ? a.threshold[H - 1 + j] : 0.f;
            mu[j] = a.centroid[H + j];
        }
    }
};

template <int B>
__device__ __forceinline__ float mag_search(float az, const MagTab<B>& tb, float (&g)[B > 1 ? B - 1 : 1]) {
    const float* tau = tb.tau;
    const float* mu = tb.mu;
    if constexpr (B == 1) {
        g[0] = 0.f;
        return mu[0];
    } else if constexpr (B == 2) {
        g[0] = az - tau[1];
        // [g >= 0] as 0 or 1 on the FMA pipe: tau[1] = 0.98..., so a negative
        // g is at least 2^-25 below 0 (exact difference near tau, or below
        // -tau/2), and g * 2^32 + 1 saturates to exactly 0 or 1.
        const float s = __saturatef(fmaf(g[0], 0x1p32f, 1.0f));
        return fmaf(s, mu[1] - mu[0], mu[0]);
    } else if constexpr (B == 3) {
        g[1] = az - tau[2];
        const bool m1 = g[1] >= 0.f;
        g[0] = az - (m1 ? tau[3] : tau[1]);
        const bool m0 = g[0] >= 0.f;
        const float hi = m0 ? mu[3] : mu[2];
        const float lo = m0 ? mu[1] : mu[0];
        return m1 ? hi : lo;
    } else {
        g[2] = az - tau[4];
        const bool m2 = g[2] >= 0.f;
        g[1] = az - (m2 ? tau[6] : tau[2]);
        const bool m1 = g[1] >= 0.f;
        const float t_hi = m2 ? tau[7] : tau[3];
        const float t_lo = m2 ? tau[5] : tau[1];
        g[0] = az - (m1 ? t_hi : t_lo);
        const bool m0 = g[0] >= 0.f;
        const float a3 = m0 ? mu[7] : mu[6], a2 = m0 ? mu[5] : mu[4];
        const float a1 = m0 ? mu[3] : mu[2], a0 = m0 ? mu[1] : mu[0];
        const float hi = m1 ? a3 : a2;
        const float lo = m1 ? a1 : a0;
        return m2 ? hi : lo;
    }
}

// z = v * inv; Lloyd-Max codes into bit planes; v <- r = z - c[code];
// returns ||r||^2.  Bit planes: the top plane is [z >= 0]; plane p < B-1 is
// bit p of the code, which equals (magnitude-index bit p) XNOR (sign), so
// every plane is assembled from sign bits with one funnel shift per
// coordinate.  Coordinates go from high to low within each 32-bit word.
template <int NV, int B>
__device__ __forceinline__ float codes_and_residual(float2 (&v)[NV / 2], float inv, const QuantArgs& a,
                                                     uint32_t (&planes)[B][NV / 32]) {
    constexpr int NG = B > 1 ? B - 1 : 1;
    const float2 inv2 = make_float2(inv, inv);
    const float2 m1 = make_float2(-1.f, -1.f);
    float2 rr = make_float2(0.f, 0.f);
    const MagTab<B> tab(a);
#pragma unroll
    for (int w = 0; w < NV / 32; ++w) {
        // four independent chains of 8 coordinates (one byte each) per plane
        uint32_t wz[4], wg[NG][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            wz[q] = 0;
#pragma unroll
            for (int p = 0; p < NG; ++p) wg[p][q] = 0;
        }
#pragma unroll
        for (int kk = 3; kk >= 0; --kk) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int k = w * 16 + q * 4 + kk;  // pair index: coordinates 2k, 2k+1
                const float2 z = __fmul2_rn(v[k], inv2);
                float g1[NG], g0[NG];
                const float mu1 = mag_search<B>(fabsf(z.y), tab, g1);
                const float mu0 = mag_search<B>(fabsf(z.x), tab, g0);
                wz[q] = push_sign(push_sign(wz[q], z.y), z.x);
                if (B > 1) {
#pragma unroll
                    for (int p = 0; p < NG; ++p) wg[p][q] = push_sign(push_sign(wg[p][q], g1[p]), g0[p]);
                }
                const float2 c = make_float2(copysignf(mu0, z.x), copysignf(mu1, z.y));
                const float2 r = __ffma2_rn(c, m1, z);
                rr = __ffma2_rn(r, r, rr);
                v[k] = r;
            }
        }
        const uint32_t z32 = wz[0] | (wz[1] << 8) | (wz[2] << 16) | (wz[3] << 24);
        planes[B - 1][w] = ~z32;
#pragma unroll
        for (int p = 0; p < B - 1; ++p)
            planes[p][w] = ~(z32 ^ (wg[p][0] | (wg[p][1] << 8) | (wg[p][2] << 16) | (wg[p][3] << 24)));
    }
    return rr.x + rr.y;
}

// Residual (2*NP coordinates) as one fp16 term into tensor memory from
// column t_hi (two fp16 per 32-bit column, even coordinate in the low half).
// S is exact in fp16 and r is rounded once, so (S r)_i carries an error of
// about 2e-4 ||r|| (fp32 accumulation): a sign can differ from the exact one
// outside a 1e-3 ||r|| band only through a 5-sigma error, ~1e-11 per bit.
template <int NP>
__device__ __forceinline__ void store_residual_tmem(const float2 (&v)[NP], uint32_t t_hi) {
#pragma unroll
    for (int cc = 0; cc < NP / 32; ++cc) {
        uint32_t hi[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const __half2 hh = __float22half2_rn(v[32 * cc + i]);
            hi[i] = *reinterpret_cast<const uint32_t*>(&hh);
        }
        tmem_st32(t_hi + cc * 32, hi);
    }
}

// Sign bits of NV accumulator columns of this thread's TMEM lane: 32-column
// loads, one wait per 64 columns, four independent 8-bit chains per word.
template <int NV, int PER_WAIT = 2>
__device__ __forceinline__ void qjl_bits_from_tmem(uint32_t taddr, uint32_t (&qw)[NV / 32]) {
#pragma unroll
    for (int cc = 0; cc < NV / 32; cc += PER_WAIT) {
        uint32_t u[PER_WAIT][32];
#pragma unroll
        for (int h = 0; h < PER_WAIT; ++h) tmem_ld32(taddr + (cc + h) * 32, u[h]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < PER_WAIT; ++h) {
            uint32_t b[4] = {0, 0, 0, 0};
#pragma unroll
            for (int i = 7; i >= 0; --i)
#pragma unroll
                for (int q = 0; q < 4; ++q) b[q] = __funnelshift_l(u[h][8 * q + i], b[q], 1);
            qw[cc + h] = ~(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24));  // bit = [u >= 0]
        }
    }
}

// Issue the QJL MMAs of one tile: acc(128 x N) = A S^T, A the fp16 residual.
// K = KD coordinates, S resident in shared memory as KD/64 K-chunks of
// N rows x 128 bytes (128-byte swizzle).
template <int N, int KD>
__device__ __forceinline__ void issue_qjl_mma(uint32_t acc, uint32_t a_hi, uint32_t s_smem) {
    constexpr uint32_t idesc = idesc_f16_f32(kTileRows, N);
#pragma unroll
    for (int ks = 0; ks < KD / 16; ++ks) {
        const uint32_t boff = (ks / 4) * (N * 128) + (ks % 4) * 32;
        const uint64_t bd = smem_desc_sw128(s_smem + boff);
        mma_f16_ts(acc, a_hi + ks * 8, bd, idesc, ks ? 1u : 0u);
    }
}

// 32 x 32 bit transpose across the warp: lane i enters with row i (bit j =
// column j) and leaves with column i (bit j = row j).  Five stages of a
// shuffle exchanging the off-diagonal sub-blocks.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const uint32_t m = s == 16 ? 0x0000FFFFu : s == 8 ? 0x00FF00FFu : s == 4 ? 0x0F0F0F0Fu : s == 2 ? 0x33333333u
                                                                                                  : 0x55555555u;
        const uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, s);
        x = (lane & s) ? ((x & ~m) | ((y >> s) & m)) : ((x & m) | ((y << s) & ~m));
    }
    return x;
}

// Block-32 store of NW words per lane: the warp holds 32 consecutive vectors
// (lane = vector); word w covers coordinates (or QJL rows) 32w .. 32w+31.
// dst points at the block's word for coordinate 0; lane i writes
// coordinate 32w + i.  Called by the whole warp.
template <int NW>
__device__ __forceinline__ void store_block32(uint32_t* dst, const uint32_t* words, uint32_t mask, int lane,
                                              bool store) {
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const uint32_t t = warp_transpose32(words[w] & mask, lane);
        if (store) dst[32 * w + lane] = t;
    }
}

template <int NWORDS>
__device__ __forceinline__ void store_words(uint32_t* dst, const uint32_t* src, uint32_t mask) {
    if (NWORDS % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NWORDS; i += 4)
            *reinterpret_cast<uint4*>(dst + i) =
                make_uint4(src[i] & mask, src[i + 1] & mask, src[i + 2] & mask, src[i + 3] & mask);
    } else {
#pragma unroll
        for (int i = 0; i < NWORDS; i += 2)
            *reinterpret_cast<uint2*>(dst + i) = make_uint2(src[i] & mask, src[i + 1] & mask);
    }
}

__device__ __forceinline__ void flag_norm(float ss, float nrm, uint32_t* status) {
    if (!(ss < INFINITY)) atomicOr(status, kStatusNonFinite);
    else if (nrm > 65504.f) atomicOr(status, kStatusNormOverflow);
}

template <int D, int B, bool QJL, int DT, bool NSN>
__global__ void __launch_bounds__(256, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap map, const __grid_constant__ QuantArgs a) {
    using C = QCfg<D, B, QJL, DT, NSN>;
    constexpr int kStages = C::kStages;
    constexpr int kWpp = D / 32;  // words per plane (whole vector)

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage0 = smem;
    uint8_t* sS = smem + kStages * C::kStageBytes;
    uint8_t* aux = sS + C::kSBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(aux);   // [4]
    uint64_t* mmadone = full + 4;                          // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mmadone + 2);
    float* xch = reinterpret_cast<float*>(aux + 256);      // [2][128] floats
    __half* so16 = reinterpret_cast<__half*>(aux + 256 + 1024);  // [2][128]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t G = gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        mbar_init(&mmadone[0], 1);
        mbar_init(&mmadone[1], 1);
        fence_mbar_init();
    }
    if (QJL) {
        // S (m = D rows, K = D) into shared memory, K-major, 128-byte swizzle:
        // K-chunk kc (64 fp16) of row n at sS + kc*D*128 + n*128, 16-byte
        // chunk c stored at position c ^ (n & 7).
        const uint4* gS = reinterpret_cast<const uint4*>(a.S);
        for (int e = tid; e < D * D / 8; e += C::kThreads) {
            const int n = e / (D / 8), cc = e % (D / 8);
            const int kc = cc / 8, c16 = cc % 8;
            *reinterpret_cast<uint4*>(sS + kc * (D * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) = gS[e];
        }
        fence_proxy_async_smem();
        if (warp == 0) {
            tmem_alloc(tmem_slot, C::kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
    }
    __syncthreads();
    uint32_t tmem = 0;
    if (QJL) {
        tc_fence_after();
        tmem = *tmem_slot;
    }

    // Stage refill: tile i lives in stage i % kStages; the leader of the
    // warpgroup that consumes it arms the stage's barrier and issues the TMA.
    auto issue_tile = [&](int64_t i) {
        const int64_t tile = blockIdx.x + i * G;
        if (tile >= a.ntiles) return;
        const int st = static_cast<int>(i % kStages);
        mbar_arrive_expect_tx(&full[st], C::kStageBytes);
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box)
            tma_load_2d(stage0 + st * C::kStageBytes + box * C::kBoxBytes, &map, &full[st], box * C::kBoxCols,
                        static_cast<int>(tile * kTileRows));
    };
    if (!C::kCoop) {
        // ---------------- compute warpgroup w: one vector per thread ----------------
        const int w = warp >> 2;
        const int r = tid & 127;
        const uint32_t bar_id = 1 + w;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tb = tmem + w * (2 * D);  // A (fp16 pairs) @ +0, acc @ +D
        if (r == 0) {
            prefetch_tmap(&map);
            for (int64_t i = w; i < kStages; i += 2) issue_tile(i);
        }
        int64_t jlocal = 0;
        int64_t i = w;
        // Epilogue state of the tile whose QJL MMA is in flight.
        bool pend = false, pend_valid = false;
        int64_t pend_vidx = 0, pend_tile = 0;
        uint32_t pend_zmask = 0, pend_parity = 0;
        auto finish_pending = [&]() -> bool {
            const bool okm = mbar_wait(&mmadone[w], pend_parity, a.status);
            if (named_bar_or(bar_id, 128, !okm)) return false;
            tc_fence_after();
            uint32_t qw[kWpp];
            qjl_bits_from_tmem<D, 1>(tb + lane_base + D, qw);
            tc_fence_before();
            if (a.layout == 0) {
                if (pend_valid) store_words<kWpp>(a.qjl + pend_vidx * kWpp, qw, pend_zmask);
            } else {
                const int64_t blk = pend_tile * 4 + (warp & 3);
                store_block32<kWpp>(a.qjl + blk * D, qw, pend_valid ? pend_zmask : 0u, lane, blk * 32 < a.n);
            }
            pend = false;
            return true;
        };
        for (;; i += 2, ++jlocal) {
            const int64_t tile = blockIdx.x + i * G;
            if (tile >= a.ntiles) break;
            const int st = static_cast<int>(i % kStages);
            const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((i / kStages) & 1), a.status);
            if (named_bar_or(bar_id, 128, !ok)) break;
            const uint8_t* sp = stage0 + st * C::kStageBytes;
            const int64_t vidx = tile * kTileRows + r;
            const bool valid = vidx < a.n;

            float2 v[D / 2];
            float nx = 0.f, nrm;
            if (NSN) {
                load_row<D, DT, false>(sp, r, v, a.pair_sign);
                const float ss = sumsq(v);
                nx = sqrtf(ss);
                flag_norm(ss, nx, a.status);
                const float inv = nx > 0.f ? sqrtf(static_cast<float>(D)) / nx : 0.f;
                xch[w * 128 + r] = inv;
                named_bar_sync(bar_id, 128);
                if (r < D) {
                    // block mean of u = sqrt(D) x / ||x|| on channel j = r
                    const int j = r;
                    float acc = 0.f;
                    for (int t = 0; t < kTileRows; ++t) {
                        float xt;
                        if (DT == DT_F32) {
                            const uint8_t* p = sp + (j / 32) * 16384 + t * 128 + ((((j % 32) / 4) ^ (t & 7)) << 4) + (j % 4) * 4;
                            xt = *reinterpret_cast<const float*>(p);
                        } else {
                            const uint8_t* p = sp + (j / 64) * 16384 + t * 128 + ((((j % 64) / 8) ^ (t & 7)) << 4) + (j % 8) * 2;
                            const uint16_t hv = *reinterpret_cast<const uint16_t*>(p);
                            xt = (DT == DT_BF16) ? u2f(static_cast<uint32_t>(hv) << 16)
                                                 : __half2float(*reinterpret_cast<const __half*>(&hv));
                        }
                        acc = fmaf(xt, xch[w * 128 + t], acc);
                    }
                    const __half o16 = __float2half_rn(acc * (1.0f / kTileRows));
                    so16[w * 128 + j] = o16;
                    a.block_mean[tile * D + j] = o16;
                }
                named_bar_sync(bar_id, 128);
                if (r == 0) issue_tile(i + kStages);
                // w = u - fp16(o), then the Rademacher signs
                const float2 inv2 = make_float2(inv, inv);
                const __half2* o2 = reinterpret_cast<const __half2*>(so16 + w * 128);
#pragma unroll
                for (int k = 0; k < D / 2; ++k) {
                    const float2 wv = __ffma2_rn(v[k], inv2, __half22float2(__hneg2(o2[k])));
                    const uint32_t ps = a.pair_sign[k];
                    v[k] = make_float2(u2f(f2u(wv.x) ^ (ps << 16)), u2f(f2u(wv.y) ^ (ps & 0x80000000u)));
                }
                nrm = sqrtf(sumsq(v));
            } else {
                load_row<D, DT, true>(sp, r, v, a.pair_sign);
                named_bar_sync(bar_id, 128);
                if (r == 0) issue_tile(i + kStages);
                const float ss = sumsq(v);
                nrm = sqrtf(ss);
                flag_norm(ss, nrm, a.status);
            }

            fwht<D / 2>(v);
            const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
            uint32_t planes[B][kWpp];
            const float rr = codes_and_residual<D, B>(v, inv, a, planes);
            const uint32_t zmask = nrm > 0.f ? 0xFFFFFFFFu : 0u;

            if (a.layout == 0) {
                if (valid) {
                    uint32_t* cp = a.codes + vidx * (B * kWpp);
#pragma unroll
                    for (int p = 0; p < B; ++p) store_words<kWpp>(cp + p * kWpp, planes[p], zmask);
                }
            } else {
                const int64_t blk = tile * 4 + (warp & 3);
                const uint32_t m = valid ? zmask : 0u;
#pragma unroll
                for (int p = 0; p < B; ++p)
                    store_block32<kWpp>(a.codes + (blk * B + p) * D, planes[p], m, lane, blk * 32 < a.n);
            }
            if (valid) {
                const float g = nrm > 0.f ? sqrtf(rr) : 0.f;
                a.norms[vidx] = __halves2half2(__float2half_rn(NSN ? nx : nrm), __float2half_rn(NSN ? nrm : g));
            }
            if (QJL) {
                // Software pipeline: the MMA of the previous tile ran while this
                // tile was computed; finish its epilogue now, which also frees the
                // A and accumulator columns for this tile.
                if (pend && !finish_pending()) break;
                store_residual_tmem<D / 2>(v, tb + lane_base);
                tmem_wait_st();
                tc_fence_before();
                named_bar_sync(bar_id, 128);
                if (r == 0) {
                    tc_fence_after();
                    issue_qjl_mma<D, D>(tb + D, tb, smem_u32(sS));
                    mma_commit(&mmadone[w]);
                }
                pend = true;
                pend_tile = tile;
                pend_vidx = vidx;
                pend_valid = valid;
                pend_zmask = zmask;
                pend_parity = static_cast<uint32_t>(jlocal & 1);
            }
        }
        if (QJL && pend) finish_pending();
        if (r == 0) {
            // Loads issued for tiles i, i+2, ... (< i + kStages) that were not consumed.
            for (int64_t k = i; k <= i + kStages; k += 2)
                if (blockIdx.x + k * G < a.ntiles)
                    mbar_wait(&full[k % kStages], static_cast<uint32_t>((k / kStages) & 1), a.status);
        }
    } else {
        // ---------------- D = 256: both warpgroups on one tile, two threads per vector ----------------
        const int h = warp >> 2;  // which half of the rotated vector
        const int r = tid & 127;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        if (tid == 0) {
            prefetch_tmap(&map);
            for (int64_t i = 0; i < kStages; ++i) issue_tile(i);
        }
        int64_t jlocal = 0;
        int64_t i = 0;
        for (;; ++i, ++jlocal) {
            const int64_t tile = blockIdx.x + i * G;
            if (tile >= a.ntiles) break;
            const int st = static_cast<int>(i % kStages);
            const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((i / kStages) & 1), a.status);
            if (named_bar_or(3, 256, !ok)) break;
            const uint8_t* sp = stage0 + st * C::kStageBytes;
            const int64_t vidx = tile * kTileRows + r;
            const bool valid = vidx < a.n;

            float2 v[64];
            const float ss = load_row_coop<DT>(sp, r, h, v, a.pair_sign);
            named_bar_sync(3, 256);
            if (tid == 0) issue_tile(i + kStages);
            const float nrm = sqrtf(ss);
            if (h == 0) flag_norm(ss, nrm, a.status);
            fwht<64>(v);
            const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
            uint32_t planes[B][4];
            const float rr = codes_and_residual<128, B>(v, inv, a, planes);
            const uint32_t zmask = nrm > 0.f ? 0xFFFFFFFFu : 0u;
            xch[h * 128 + r] = rr;
            if (QJL) {
                // A columns [0,128) (two fp16 per column), acc [256,512)
                store_residual_tmem<64>(v, tmem + lane_base + h * 64);
                tmem_wait_st();
                tc_fence_before();
            }
            named_bar_sync(3, 256);
            if (QJL && tid == 0) {
                tc_fence_after();
                issue_qjl_mma<256, 256>(tmem + 256, tmem, smem_u32(sS));
                mma_commit(&mmadone[0]);
            }
            if (a.layout == 0) {
                if (valid) {
                    uint32_t* cp = a.codes + vidx * (B * 8) + h * 4;
#pragma unroll
                    for (int p = 0; p < B; ++p) store_words<4>(cp + p * 8, planes[p], zmask);
                }
            } else {
                const int64_t blk = tile * 4 + (warp & 3);
#pragma unroll
                for (int p = 0; p < B; ++p)
                    store_block32<4>(a.codes + (blk * B + p) * 256 + h * 128, planes[p], valid ? zmask : 0u, lane,
                                     blk * 32 < a.n);
            }
            if (valid && h == 0) {
                const float g = nrm > 0.f ? sqrtf(xch[r] + xch[128 + r]) : 0.f;
                a.norms[vidx] = __halves2half2(__float2half_rn(nrm), __float2half_rn(g));
            }
            if (QJL) {
                const bool okm = mbar_wait(&mmadone[0], static_cast<uint32_t>(jlocal & 1), a.status);
                if (named_bar_or(3, 256, !okm)) break;
                tc_fence_after();
                uint32_t qw[4];
                qjl_bits_from_tmem<128>(tmem + lane_base + 256 + h * 128, qw);
                tc_fence_before();
                if (a.layout == 0) {
                    if (valid) store_words<4>(a.qjl + vidx * 8 + h * 4, qw, zmask);
                } else {
                    const int64_t blk = tile * 4 + (warp & 3);
                    store_block32<4>(a.qjl + blk * 256 + h * 128, qw, valid ? zmask : 0u, lane, blk * 32 < a.n);
                }
            }
            // xch is rewritten next tile only after this barrier
            named_bar_sync(3, 256);
        }
        if (tid == 0) {
            for (int64_t k = i; k <= i + kStages; ++k)
                if (blockIdx.x + k * G < a.ntiles)
                    mbar_wait(&full[k % kStages], static_cast<uint32_t>((k / kStages) & 1), a.status);
        }
    }

    __syncthreads();
    if (QJL && warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D, int B, bool QJL, int DT, bool NSN>
cudaError_t launch_quantize_t(const CUtensorMap& map, const QuantArgs& a, int num_sms, cudaStream_t s) {
    using C = QCfg<D, B, QJL, DT, NSN>;
    auto kern = quantize_kernel<D, B, QJL, DT, NSN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t grid = a.ntiles < num_sms ? a.ntiles : num_sms;
    if (grid <= 0) return cudaSuccess;
    kern<<<static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace kvq
