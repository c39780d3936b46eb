// quantize_tc.cuh -- the quantize kernel (and its NSN front end) with the
// rotation on the tensor cores, for 16-bit input: d <= 128, and d = 256
// without QJL.
//
// Method (TurboQuant blog, "Estagio 1" and "Estagio 2"; PolarQuant section 2),
// per vector x: y = H (delta .* x) (unnormalised Sylvester Hadamard, so
// ||y||^2 = d ||x||^2), n = ||x||, z = y / n, code_j = #{k : z_j >= t_k},
// r = z - c[code], gamma = ||r||, QJL bits = [S r >= 0], norms fp16.
//
// Design (sm_100a):
// * The randomized Hadamard rotation is one dense product per 128-vector
//   tile, Y(128 x d) = X(128 x d) (H D)^T, on tcgen05: X straight from the
//   TMA stage (K-major, 128-byte swizzle), H D (entries +-1, exact in bf16
//   and fp16, built in shared memory at start-up) as the B operand, fp32
//   accumulation into tensor memory.  Every product x_k * (+-1) is exact,
//   so y carries only fp32 summation rounding.
// * Four warpgroups per CTA (one CTA per SM), each owning 128 TMEM columns
//   and whole tiles; a thread owns one vector (its TMEM lane).  Each stage of
//   the x ring belongs to one warpgroup; it is free as soon as the rotation
//   MMA has read it, and the warpgroup refills it then.
// * d = 256 (no QJL: S would not fit beside the stages): H of order 256 is
//   [[H', H'], [H', -H']] with H' of order 128, so the rotation is two
//   products P = X1 (H' D1)^T and Q = X2 (H' D2)^T over the two halves of x
//   (64 KB of B operands instead of 128 KB), and the passes read
//   y = (P + Q, P - Q) group by group.  Two warpgroups of 256 columns each,
//   two 64 KB stages.
// * Pass 1 reads y back (32 columns at a time) for ||y||^2; pass 2 reads it
//   again, forms codes and the residual chunk by chunk and writes the fp16
//   residual into the already consumed columns [0, d/2).
// * QJL: U(128 x 64) = R S_h^T for the two 64-row halves of S (d = 128; one
//   half for d = 64), accumulated in columns [64, 128), and the sign bits are
//   packed from there.  The residual enters as one fp16 term: with S exact in
//   fp16 and fp32 accumulation the error of (S r)_i is about 2e-4 ||r|| (one
//   standard deviation), so a sign can differ from the exact one only where
//   |(S r)_i| is a few 1e-4 ||r||, inside the 1e-3 ||r|| band where the sign
//   is not pinned (a flip outside it needs a 5-sigma error, ~1e-11 per bit).
// * NSN front end ([NSN] "NSNQuant" sections 1-2): the tile is one block of
//   128 tokens; sc = sqrt(d)/||x|| from the staged tile, the channel means
//   of u = sc x and their fp16 rounding o, and ho = H (delta .* o) by a
//   one-warp FWHT; the rotation of w = u - o is then sc y - ho.
// * Every mbarrier wait is bounded and its outcome agreed on by the
//   warpgroup; loads still in flight at exit are waited for.
#pragma once

#include "quantize.cuh"

namespace kvq {

template <int D, bool QJL, bool NSN = false>
struct TcCfg {
    static constexpr int kTileBytes = kTileRows * D * 2;   // 16-bit input
    static constexpr int kBoxBytes = 128 * kTileRows;      // 64 elements x 128 rows
    static constexpr int kBoxes = D * 2 / 128;
    // The rotation is kNMat products of N = K = kNB: at d = 256 the two
    // 128-coordinate halves x1, x2 of x give P = (H D1) x1 and Q = (H D2) x2
    // (H of order 128, D1, D2 the two halves of the sign diagonal), and the
    // Sylvester recursion puts the rotated vector together as (P + Q, P - Q).
    static constexpr int kNB = D > 128 ? 128 : D;
    static constexpr int kNMat = D / kNB;
    static constexpr int kMatBytes = kNMat * kNB * kNB * 2;  // H D blocks, 16-bit, K-major, swizzled
    static constexpr int kSBytes = QJL ? D * D * 2 : 0;      // S, same layout
    static constexpr int kCols = D > 128 ? 256 : 128;        // tensor-memory columns per warpgroup
    static constexpr int kWG = 512 / kCols;
    static constexpr int kThreads = 128 * kWG;
    // NSN scratch floats per warpgroup: scale [128], mean [D], rotated mean [D],
    // partial channel sums [1024], reductions [8]
    static constexpr int kNsnF = 1160 + 2 * D;
    static constexpr int kAuxBytes = NSN ? 24576 : 1024;
    static constexpr int kBudget = 225 * 1024;
    static constexpr int kStagesRaw = (kBudget - kMatBytes - kSBytes - kAuxBytes) / kTileBytes;
    // Tile i goes to warpgroup i % kWG and stage i % kStages; with kStages a
    // multiple of kWG every stage belongs to one warpgroup, which consumes its
    // phases strictly in order (a parity wait can never see a stale phase).
    static constexpr int kStages = (kStagesRaw > 8 ? 8 : kStagesRaw) / kWG * kWG;
    static constexpr int kSmemBytes = 1024 + kStages * kTileBytes + kMatBytes + kSBytes + kAuxBytes;
    static constexpr int kQN = 64;                          // rows of S per QJL MMA
    static_assert(D == 64 || D == 128 || (D == 256 && !QJL), "tensor-core rotation: d in {64, 128}, or 256 without QJL");
    static_assert(kStages >= kWG, "one stage per warpgroup at least");
    static_assert(1024 + kWG * kNsnF * 4 <= kAuxBytes || !NSN, "NSN scratch");
};

// Column order of the rotated vector and of the residual in tensor memory.
// Within each group of 32 columns, column 32c + 2i + e holds coordinate
// 32c + i + 16e (i < 16, e in {0, 1}).  A register pair (2i, 2i + 1) of a
// 32-column load then holds coordinates i and i + 16 of the group, so the
// packed fp32x2 operations act on the two 16-bit halves of a packed word and
// every plane word is two 16-bit chains joined by one byte permute.  The
// rotation matrix's rows and the residual's K order (S's columns) follow the
// same permutation, so the products are unchanged.
__host__ __device__ constexpr int col_coord(int col) { return (col & ~31) + ((col & 31) >> 1) + ((col & 1) << 4); }

// Sign word of 32 accumulator values: bit i = [u_i >= 0] (two 16-bit chains).
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&u)[32]) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 15; i >= 0; --i) {
        lo = __funnelshift_l(u[i], lo, 1);
        hi = __funnelshift_l(u[16 + i], hi, 1);
    }
    return ~__byte_perm(lo, hi, 0x5410);
}

// Per-lane constants of the 32 x 32 bit transpose (bit_transpose32).
struct Transpose32 {
    uint32_t sel16, sel8;      // byte selectors of the 16- and 8-bit stages
    uint32_t rot[3], keep[3];  // rotate amount and kept-bit mask of the 4-, 2- and 1-bit stages
    __device__ __forceinline__ explicit Transpose32(int lane) {
        sel16 = (lane & 16) ? 0x3276u : 0x5410u;
        sel8 = (lane & 8) ? 0x3715u : 0x6240u;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int s = 4 >> k;
            const uint32_t m = k == 0 ? 0x0F0F0F0Fu : (k == 1 ? 0x33333333u : 0x55555555u);
            const bool hi = (lane & s) != 0;
            rot[k] = hi ? 32u - s : static_cast<uint32_t>(s);
            keep[k] = hi ? ~m : m;
        }
    }
};

// 32 x 32 bit transpose across the warp: lane i enters with row i (bit j =
// column j) and leaves with column i (bit j = row j).  Each of the five
// stages swaps the off-diagonal s x s blocks with the partner lane i ^ s:
// one shuffle, then a byte permute (s = 16, 8) or a rotate and a bit select
// (s = 4, 2, 1; the bits rotated around the word land in positions the
// select does not keep).
__device__ __forceinline__ uint32_t bit_transpose32(uint32_t x, const Transpose32& t) {
    uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, 16);
    x = __byte_perm(x, y, t.sel16);
    y = __shfl_xor_sync(0xFFFFFFFFu, x, 8);
    x = __byte_perm(x, y, t.sel8);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        y = __shfl_xor_sync(0xFFFFFFFFu, x, 4 >> k);
        const uint32_t r = __funnelshift_l(y, y, t.rot[k]);
        x = (x & t.keep[k]) | (r & ~t.keep[k]);
    }
    return x;
}

// Block-32 store of NW words per lane (lane = vector of the block of 32):
// lane i writes the transposed word of coordinate (or QJL row) 32w + i.
template <int NW>
__device__ __forceinline__ void store_block32_t(uint32_t* dst, const uint32_t* words, uint32_t mask, int lane,
                                                bool store) {
    const Transpose32 t(lane);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const uint32_t x = bit_transpose32(words[w] & mask, t);
        if (store) dst[32 * w + lane] = x;
    }
}

// Codebook constants of the coding pass for B bits (symmetric codebook,
// H = 2^(B-1) levels per sign): the positive decision levels tau_1..tau_{H-1}
// (tau_j = t[H-1+j]) and the centroid magnitudes mu_0..mu_{H-1}.  The
// magnitude index idx = #{j : |z| >= tau_j} is found by a binary search
// whose bit at each level is s = sat(g * K + 1) with g = |y| - (level) * n:
// exactly 0 or 1, since a nonzero g is at least |y| 2^-24 (the two terms are
// within a factor of two near a level) and K = 2^40 / n.  The level of the
// next step and mu_idx are multilinear in the bits found, so they are fused
// multiply-adds on the FMA pipe (no branch, select or indexed load).
template <int B>
struct CodeTab {
    static constexpr int H = 1 << (B - 1);
    float lev[H > 1 ? H - 1 : 1];  // multilinear coefficients of the levels (times n per vector)
    float mu[H];                   // multilinear coefficients of mu_idx
    __device__ __forceinline__ explicit CodeTab(const QuantArgs& a) {
        float tau[H], m[H];
#pragma unroll
        for (int j = 0; j < H; ++j) {
            tau[j] = j > 0 ? a.threshold[H - 1 + j] : 0.f;
            m[j] = a.centroid[H + j];
        }
        if constexpr (B == 1) {
            lev[0] = 0.f;
            mu[0] = m[0];
        } else if constexpr (B == 2) {
            lev[0] = tau[1];
            mu[0] = m[0];
            mu[1] = m[1] - m[0];
        } else if constexpr (B == 3) {
            lev[0] = tau[2];                              // level 1
            lev[1] = tau[1];                              // level 2: tau_1 + s1 (tau_3 - tau_1)
            lev[2] = tau[3] - tau[1];
            mu[0] = m[0];                                 // mu = s0 (s1 X + a1) + (s1 (m2 - m0) + m0)
            mu[1] = m[1] - m[0];
            mu[2] = m[2] - m[0];
            mu[3] = m[3] - m[2] - m[1] + m[0];
        } else {
            lev[0] = tau[4];                              // level 1
            lev[1] = tau[2];                              // level 2: tau_2 + s2 (tau_6 - tau_2)
            lev[2] = tau[6] - tau[2];
            lev[3] = tau[1];                              // level 3: tau_1 + s1 (tau_3 - tau_1)
            lev[4] = tau[3] - tau[1];                     //   + s2 (tau_5 - tau_1) + s1 s2 X
            lev[5] = tau[5] - tau[1];
            lev[6] = tau[7] - tau[5] - tau[3] + tau[1];
            // mu = s0 A(s1, s2) + Bv(s1, s2), A and Bv bilinear
            mu[0] = m[0];
            mu[1] = m[2] - m[0];
            mu[2] = m[4] - m[0];
            mu[3] = m[6] - m[4] - m[2] + m[0];
            const float a0 = m[1] - m[0], a2 = m[3] - m[2], a4 = m[5] - m[4], a6 = m[7] - m[6];
            mu[4] = a0;
            mu[5] = a2 - a0;
            mu[6] = a4 - a0;
            mu[7] = a6 - a4 - a2 + a0;
        }
    }
};

// Per-vector constants: 1/n, K = 2^40/n and the levels scaled by n.
template <int B>
struct VecTab {
    float2 inv2;
    float K;
    float lev[CodeTab<B>::H > 1 ? CodeTab<B>::H - 1 : 1];
    __device__ __forceinline__ VecTab(const CodeTab<B>& c, float nrm, float inv) {
        inv2 = make_float2(inv, inv);
        // (bounded so that a vector whose norm is below 2^-86 -- stored as an fp16
        // norm of 0 -- cannot make it overflow)
        K = fminf(inv * 0x1p40f, 0x1p126f);
#pragma unroll
        for (int j = 0; j < (CodeTab<B>::H > 1 ? CodeTab<B>::H - 1 : 1); ++j) lev[j] = c.lev[j] * nrm;
    }
};

__device__ __forceinline__ float2 sat_bits(float2 y, float level, float K) {
    return make_float2(__saturatef(fmaf(fabsf(y.x) - level, K, 1.0f)), __saturatef(fmaf(fabsf(y.y) - level, K, 1.0f)));
}
__device__ __forceinline__ float2 sat_bits2(float2 y, float2 level, float K) {
    return make_float2(__saturatef(fmaf(fabsf(y.x) - level.x, K, 1.0f)),
                       __saturatef(fmaf(fabsf(y.y) - level.y, K, 1.0f)));
}
__device__ __forceinline__ float2 f2s(float v) { return make_float2(v, v); }

// Codes and residual of one 32-column group of this thread's vector.
// v[i] = (y of coordinate i, y of coordinate 16 + i) of the group (column
// order above); y = H D x unnormalised, n = ||x||.  Out: the B plane words of
// the group (token layout: bit i = coordinate i of the group), the fp16
// residual r = y/n - c[code] as 16 packed pairs (pair i = coordinates i and
// 16 + i), and ||r||^2 accumulated into rr.
// Plane words: the top plane is [y >= 0]; plane p < B-1 is bit p of the code,
// which is (magnitude-index bit p) XOR (sign bit of y).
template <int B>
__device__ __forceinline__ void code_group(const float2 (&v)[16], const CodeTab<B>& ct, const VecTab<B>& vt,
                                           uint32_t (&hres)[16], uint32_t (&words)[B], float2& rr) {
    constexpr int NB = B > 1 ? B - 1 : 1;
    uint32_t sl = 0, sh = 0;
    float2 acc[NB];
#pragma unroll
    for (int p = 0; p < NB; ++p) acc[p] = make_float2(0.f, 0.f);
    const float2 two = f2s(2.0f);
#pragma unroll
    for (int i = 15; i >= 0; --i) {
        const float2 y = v[i];
        sl = push_sign(sl, y.x);
        sh = push_sign(sh, y.y);
        float2 mu;
        if constexpr (B == 1) {
            mu = f2s(ct.mu[0]);
        } else if constexpr (B == 2) {
            const float2 s0 = sat_bits(y, vt.lev[0], vt.K);
            acc[0] = __ffma2_rn(acc[0], two, s0);
            mu = __ffma2_rn(s0, f2s(ct.mu[1]), f2s(ct.mu[0]));
        } else if constexpr (B == 3) {
            const float2 s1 = sat_bits(y, vt.lev[0], vt.K);
            const float2 l2 = __ffma2_rn(s1, f2s(vt.lev[2]), f2s(vt.lev[1]));
            const float2 s0 = sat_bits2(y, l2, vt.K);
            acc[1] = __ffma2_rn(acc[1], two, s1);
            acc[0] = __ffma2_rn(acc[0], two, s0);
            const float2 hiA = __ffma2_rn(s1, f2s(ct.mu[3]), f2s(ct.mu[1]));
            const float2 loB = __ffma2_rn(s1, f2s(ct.mu[2]), f2s(ct.mu[0]));
            mu = __ffma2_rn(s0, hiA, loB);
        } else {
            const float2 s2 = sat_bits(y, vt.lev[0], vt.K);
            const float2 l2 = __ffma2_rn(s2, f2s(vt.lev[2]), f2s(vt.lev[1]));
            const float2 s1 = sat_bits2(y, l2, vt.K);
            const float2 la = __ffma2_rn(s2, f2s(vt.lev[6]), f2s(vt.lev[4]));
            const float2 lb = __ffma2_rn(s2, f2s(vt.lev[5]), f2s(vt.lev[3]));
            const float2 l3 = __ffma2_rn(s1, la, lb);
            const float2 s0 = sat_bits2(y, l3, vt.K);
            acc[2] = __ffma2_rn(acc[2], two, s2);
            acc[1] = __ffma2_rn(acc[1], two, s1);
            acc[0] = __ffma2_rn(acc[0], two, s0);
            const float2 ba = __ffma2_rn(s2, f2s(ct.mu[3]), f2s(ct.mu[1]));
            const float2 bb = __ffma2_rn(s2, f2s(ct.mu[2]), f2s(ct.mu[0]));
            const float2 bv = __ffma2_rn(s1, ba, bb);
            const float2 aa = __ffma2_rn(s2, f2s(ct.mu[7]), f2s(ct.mu[5]));
            const float2 ab = __ffma2_rn(s2, f2s(ct.mu[6]), f2s(ct.mu[4]));
            const float2 av = __ffma2_rn(s1, aa, ab);
            mu = __ffma2_rn(s0, av, bv);
        }
        // -c[code] = -(sign of y) mu (mu > 0): one bit select per coordinate
        const float2 nc = make_float2(u2f(f2u(mu.x) | (~f2u(y.x) & 0x80000000u)),
                                      u2f(f2u(mu.y) | (~f2u(y.y) & 0x80000000u)));
        const float2 r = __ffma2_rn(y, vt.inv2, nc);
        rr = __ffma2_rn(r, r, rr);
        const __half2 hh = __float22half2_rn(r);
        hres[i] = *reinterpret_cast<const uint32_t*>(&hh);
    }
    const uint32_t sw = __byte_perm(sl, sh, 0x5410);  // sign bits of y (1 = negative)
    words[B - 1] = ~sw;
#pragma unroll
    for (int p = 0; p < B - 1; ++p) {
        // the chains hold integers < 2^16: adding 2^23 puts them in the low mantissa bits
        const float2 t = __fadd2_rn(acc[p], f2s(0x1p23f));
        words[p] = __byte_perm(f2u(t.x), f2u(t.y), 0x5410) ^ sw;
    }
}

// Sum of squares of row r of a 16-bit stage (boxes of 64 elements x 128
// rows, 128-byte swizzle: 16-byte chunk c of row r at c ^ (r & 7)).
template <int D, int DT>
__device__ __forceinline__ float stage_row_sumsq(const uint8_t* sp, int r) {
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int box = 0; box < D / 64; ++box) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 q = *reinterpret_cast<const uint4*>(sp + box * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 v;
                if (DT == DT_BF16) v = make_float2(u2f(w[k] << 16), u2f(w[k] & 0xFFFF0000u));
                else v = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
                if (k & 1) a1 = __ffma2_rn(v, v, a1);
                else a0 = __ffma2_rn(v, v, a0);
            }
        }
    }
    a0 = __fadd2_rn(a0, a1);
    return a0.x + a0.y;
}

// Element (t, j) of a 16-bit stage as fp32.
template <int DT>
__device__ __forceinline__ float stage_elem(const uint8_t* sp, int t, int j) {
    const uint8_t* p = sp + (j / 64) * 16384 + t * 128 + ((((j % 64) / 8) ^ (t & 7)) << 4) + (j % 8) * 2;
    const uint16_t hv = *reinterpret_cast<const uint16_t*>(p);
    return (DT == DT_BF16) ? u2f(static_cast<uint32_t>(hv) << 16) : __half2float(*reinterpret_cast<const __half*>(&hv));
}

template <int D, int B, bool QJL, int DT, bool NSN = false, bool DQ = false>
__global__ void __launch_bounds__(TcCfg<D, QJL, NSN>::kThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap map, const __grid_constant__ CUtensorMap map1,
                       const __grid_constant__ QuantArgs a) {
    static_assert(!(NSN && QJL), "NSN front end: no QJL");
    static_assert(!DQ || NSN, "double quantization is of the NSN side data");
    using C = TcCfg<D, QJL, NSN>;
    constexpr int RB = (8 + D / 2 + 64 + 15) / 16 * 16;  // DQ: side record bytes per block
    constexpr int NS = C::kStages;
    constexpr int kWpp = D / 32;
    constexpr int NB = C::kNB;
    constexpr uint32_t kIdescH = idesc_16bit_f32(kTileRows, NB, DT == DT_BF16);
    constexpr uint32_t kIdescQ = idesc_16bit_f32(kTileRows, C::kQN, false);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage0 = smem;
    uint8_t* sHD = smem + NS * C::kTileBytes;
    uint8_t* sS = sHD + C::kMatBytes;
    uint8_t* aux = sS + C::kSBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(aux);    // [8]
    uint64_t* hbar = full + 8;                              // [4] rotation MMA done
    uint64_t* qbar = hbar + 4;                              // [4] QJL MMA done
    uint32_t* iss = reinterpret_cast<uint32_t*>(qbar + 4);  // [8] loads issued per stage
    uint32_t* con = iss + 8;                                // [8] loads consumed per stage
    uint32_t* tmem_slot = con + 8;
    float* nsn_aux = reinterpret_cast<float*>(aux + 1024);  // NSN: [warpgroups][kNsnF]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int wg = warp >> 2;
    const int r = tid & 127;
    const int64_t G = gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < 8; ++s) {
            mbar_init(&full[s], 1);
            iss[s] = 0;
            con[s] = 0;
        }
        for (int w = 0; w < 4; ++w) {
            mbar_init(&hbar[w], 1);
            mbar_init(&qbar[w], 1);
        }
        fence_mbar_init();
    }
    // Block m of H D as the B operand (row n = output column n, which holds
    // coordinate col_coord(n); K = input coordinate k of the block's half):
    // entry (n, k) = (-1)^popcount(col_coord(n) & k) delta_{m NB + k}.  K-chunk
    // kc (64 entries) of row n at sHD + m*NB*NB*2 + kc*NB*128 + n*128, 16-byte
    // chunk c at c ^ (n & 7).
    {
        const uint32_t one = (DT == DT_BF16) ? 0x3F80u : 0x3C00u;
        for (int e = tid; e < C::kNMat * NB * NB / 8; e += C::kThreads) {
            const int m = e / (NB * NB / 8), em = e % (NB * NB / 8);
            const int n = em / (NB / 8), cc = em % (NB / 8);
            const int kc = cc / 8, c16 = cc % 8;
            const int jn = col_coord(n);
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int k = 8 * cc + 2 * q;
                const uint32_t ps = a.pair_sign[(m * NB + k) >> 1];
                const uint32_t s0 = ((__popc(jn & k) & 1u) << 15) ^ (ps & 0x8000u);
                const uint32_t s1 = ((__popc(jn & (k + 1)) & 1u) << 15) ^ ((ps >> 16) & 0x8000u);
                w4[q] = (one | s0) | ((one | s1) << 16);
            }
            *reinterpret_cast<uint4*>(sHD + m * (NB * NB * 2) + kc * (NB * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    if (QJL) {
        // S (written once at handle creation, before any launch) with its
        // columns in the residual's K order: K index kk is coordinate
        // col_coord(kk), so 8 consecutive K entries are two runs of 4
        // consecutive columns of S (coordinates i.. and 16 + i..).
        const uint16_t* gS = reinterpret_cast<const uint16_t*>(a.S);
        for (int e = tid; e < D * D / 8; e += C::kThreads) {
            const int n = e / (D / 8), cc = e % (D / 8);
            const int kc = cc / 8, c16 = cc % 8;
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int kk = 8 * cc + 2 * q;
                w4[q] = static_cast<uint32_t>(gS[n * D + col_coord(kk)]) |
                        (static_cast<uint32_t>(gS[n * D + col_coord(kk + 1)]) << 16);
            }
            *reinterpret_cast<uint4*>(sS + kc * (D * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Launched as a programmatic dependent: the input may come from the grid
    // before this one, so nothing global is read or written before this.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Let the next programmatic dependent be scheduled now: its CTAs take an
    // SM as soon as one of ours exits, so their set-up overlaps our tail (it
    // still waits for this whole grid before it reads or writes memory).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Tile i (local index) lives in stage i % NS.
    auto issue_tile = [&](int64_t i) {
        const int64_t tile = blockIdx.x + i * G;
        if (tile >= a.ntiles) return;
        const bool s1 = tile >= a.ntiles0;  // second stream of vectors
        const int64_t lt = s1 ? tile - a.ntiles0 : tile;
        const int st = static_cast<int>(i % NS);
        iss[st] += 1;
        mbar_arrive_expect_tx(&full[st], C::kTileBytes);
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box)
            tma_load_2d(stage0 + st * C::kTileBytes + box * C::kBoxBytes, s1 ? &map1 : &map, &full[st], box * 64,
                        static_cast<int>(lt * kTileRows));
    };
    if (tid == 0) {
        prefetch_tmap(&map);
        if (a.ntiles0 < a.ntiles) prefetch_tmap(&map1);
        for (int64_t i = 0; i < NS; ++i) issue_tile(i);
    }
    __syncthreads();

    const uint32_t bar_id = 1 + wg;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tcol = tmem + static_cast<uint32_t>(wg * C::kCols);  // this warpgroup's columns
    const uint32_t tl = tcol + lane_base;                            // ... at this thread's lane
    uint32_t hpar = 0, qpar = 0;
    const CodeTab<B> ctab(a);

    for (int64_t i = wg;; i += C::kWG) {
        const int64_t tile_g = blockIdx.x + i * G;
        if (tile_g >= a.ntiles) break;
        // the tile's stream of vectors and its outputs
        const bool s1 = tile_g >= a.ntiles0;
        const int64_t tile = s1 ? tile_g - a.ntiles0 : tile_g;
        const int64_t n_s = s1 ? a.n1 : a.n;
        const int layout_s = s1 ? a.layout1 : a.layout;
        uint32_t* const codes_s = s1 ? a.codes1 : a.codes;
        uint32_t* const qjl_s = s1 ? a.qjl1 : a.qjl;
        __half2* const norms_s = s1 ? a.norms1 : a.norms;
        const int st = static_cast<int>(i % NS);
        const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((i / NS) & 1), a.status);
        if (named_bar_or(bar_id, 128, !ok)) break;
        if (r == 0) {
            con[st] += 1;
            // ---- rotation: Y = X (H D)^T into columns [0, D) (d = 256: P, Q) ----
            tc_fence_after();
            const uint32_t xs = smem_u32(stage0 + st * C::kTileBytes);
            // (read through an opaque move so that the B descriptors are formed
            // here, not hoisted out of the tile loop into registers held throughout)
            uint32_t hs;
            asm volatile("mov.b32 %0, %1;" : "=r"(hs) : "r"(smem_u32(sHD)));
#pragma unroll
            for (int m = 0; m < C::kNMat; ++m) {
#pragma unroll
                for (int ks = 0; ks < NB / 16; ++ks) {
                    const uint32_t aoff = (m * (NB / 64) + ks / 4) * C::kBoxBytes + (ks % 4) * 32;
                    const uint32_t boff = m * (NB * NB * 2) + (ks / 4) * (NB * 128) + (ks % 4) * 32;
                    mma_f16_ss(tcol + m * NB, smem_desc_sw128(xs + aoff), smem_desc_sw128(hs + boff), kIdescH,
                               ks > 0 ? 1u : 0u);
                }
            }
            mma_commit(&hbar[wg]);
        }
        // NSN front end on the tile (= one block of 128 tokens of one head):
        // sc = sqrt(D)/||x||, block mean o of u = sc x per channel, fp16(o),
        // and ho = H (delta .* fp16(o)), so that H D w = sc y - ho.
        float nx = 0.f, sc = 0.f;
        float* xch = nsn_aux + wg * C::kNsnF;  // [128] sc per token
        float* so = xch + 128;                  // [D] delta .* fp16(o)
        float* ho = xch + 128 + D;              // [D] H (delta .* fp16(o)), in tensor-memory column order
        float* opart = xch + 128 + 2 * D;       // [1024 / D][D] partial channel sums
        float* red = xch + 1152 + 2 * D;        // DQ: [4] block max of ||x|| / [2][4] channel min, max
        if constexpr (NSN) {
            const uint8_t* sp = stage0 + st * C::kTileBytes;
            const float ssx0 = stage_row_sumsq<D, DT>(sp, r);
            nx = sqrtf(ssx0);
            flag_norm(ssx0, nx, a.status);
            uint8_t* rec = DQ ? a.side + tile * RB : nullptr;  // DQ: this block's side record
            if constexpr (!DQ) {
                sc = nx > 0.f ? sqrtf(static_cast<float>(D)) / nx : 0.f;
            } else {
                // 4-bit norm codes on the block's step nstep = fp16(max ||x|| / 15):
                // q = 0 for a zero token, else clamp(rint(||x|| / nstep), 1, 15);
                // the transform divides by n1 = q nstep, the stored value
                float m = nx;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                if (lane == 0) red[warp & 3] = m;
                named_bar_sync(bar_id, 128);
                const float mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
                const __half ns16 = __float2half_rn(mx / 15.0f);
                const float ns = __half2float(ns16);
                int qn = 0;
                if (nx > 0.f && ns > 0.f) qn = min(max(__float2int_rn(nx / ns), 1), 15);
                sc = qn > 0 ? sqrtf(static_cast<float>(D)) / (static_cast<float>(qn) * ns) : 0.f;
                const int qp = __shfl_down_sync(0xFFFFFFFFu, qn, 1);
                if (tile * kTileRows < n_s) {
                    if ((r & 1) == 0) rec[8 + D / 2 + r / 2] = static_cast<uint8_t>(qn | (qp << 4));
                    if (r == 0) *reinterpret_cast<__half*>(rec + 4) = ns16;
                    if (r < 2) rec[6 + r] = 0;
                    if (r >= 2 && r < 2 + (RB - 8 - D / 2 - 64)) rec[8 + D / 2 + 64 + (r - 2)] = 0;
                }
            }
            xch[r] = sc;
            named_bar_sync(bar_id, 128);
            {
                // thread r: channels 8o .. 8o + 7 (one 16-byte chunk of a row) over
                // the tokens of group q; four independent fp32x2 sums
                constexpr int NO = D / 8, QG = kTileRows / NO, TPG = kTileRows / QG;
                const int o = r % NO, q = r / NO;
                const uint8_t* cb = sp + (o / 8) * 16384;
                float2 acc[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll 4
                for (int t = q * TPG; t < (q + 1) * TPG; ++t) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(cb + t * 128 + (((o % 8) ^ (t & 7)) << 4));
                    const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
                    const float sct = xch[t];
                    const float2 s2 = make_float2(sct, sct);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 xv = (DT == DT_BF16)
                                              ? make_float2(u2f(w4[k] << 16), u2f(w4[k] & 0xFFFF0000u))
                                              : __half22float2(*reinterpret_cast<const __half2*>(&w4[k]));
                        acc[k] = __ffma2_rn(xv, s2, acc[k]);
                    }
                }
                float4* dst = reinterpret_cast<float4*>(opart + q * D + 8 * o);
                dst[0] = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
                dst[1] = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
            }
            named_bar_sync(bar_id, 128);
            // thread r holds the block means of channels r + 128 k (k < kCh; r < D)
            constexpr int kCh = (D + 127) / 128;
            float om[kCh];
            if (r < D) {
                constexpr int QG = kTileRows / (D / 8);
                float mn = INFINITY, mxo = -INFINITY;
#pragma unroll
                for (int k = 0; k < kCh; ++k) {
                    const int ch = r + 128 * k;
                    float acc = 0.f;
#pragma unroll
                    for (int q = 0; q < QG; ++q) acc += opart[q * D + ch];
                    om[k] = acc * (1.0f / kTileRows);
                    if constexpr (!DQ) {
                        const __half o16 = __float2half_rn(om[k]);
                        if (tile * kTileRows < n_s) a.block_mean[tile * D + ch] = o16;
                        const uint32_t ps = a.pair_sign[ch >> 1];
                        const bool neg = ((ps >> ((ch & 1) ? 31 : 15)) & 1u) != 0;
                        so[ch] = neg ? -__half2float(o16) : __half2float(o16);
                    } else {
                        mn = fminf(mn, om[k]);
                        mxo = fmaxf(mxo, om[k]);
                    }
                }
                if constexpr (DQ) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
                        mxo = fmaxf(mxo, __shfl_xor_sync(0xFFFFFFFFu, mxo, o));
                    }
                    if (lane == 0) {
                        red[warp & 3] = mn;
                        red[4 + (warp & 3)] = mxo;
                    }
                }
            }
            if constexpr (DQ) {
                // 4-bit mean codes on [lo, lo + 15 step], lo = fp16(min o),
                // step = fp16((max o - min o) / 15); o_hat = fp32(lo + step q)
                named_bar_sync(bar_id, 128);
                if (r < D) {
                    constexpr int kMW = (D < 128 ? D : 128) / 32;  // warps holding channels
                    float lo = red[0], hi = red[4];
#pragma unroll
                    for (int w = 1; w < kMW; ++w) {
                        lo = fminf(lo, red[w]);
                        hi = fmaxf(hi, red[4 + w]);
                    }
                    const __half lo16 = __float2half_rn(lo), st16 = __float2half_rn((hi - lo) / 15.0f);
                    const float lof = __half2float(lo16), stf = __half2float(st16);
#pragma unroll
                    for (int k = 0; k < kCh; ++k) {
                        const int ch = r + 128 * k;
                        int qo = 0;
                        if (stf > 0.f) qo = min(max(__float2int_rn((om[k] - lof) / stf), 0), 15);
                        const float oh = fmaf(stf, static_cast<float>(qo), lof);
                        const int qp = __shfl_down_sync(0xFFFFFFFFu, qo, 1);
                        if (tile * kTileRows < n_s) {
                            if ((ch & 1) == 0) rec[8 + ch / 2] = static_cast<uint8_t>(qo | (qp << 4));
                            if (ch == 0) {
                                *reinterpret_cast<__half*>(rec) = lo16;
                                *reinterpret_cast<__half*>(rec + 2) = st16;
                            }
                        }
                        const uint32_t ps = a.pair_sign[ch >> 1];
                        const bool neg = ((ps >> ((ch & 1) ? 31 : 15)) & 1u) != 0;
                        so[ch] = neg ? -oh : oh;
                    }
                }
            }
            named_bar_sync(bar_id, 128);
            if ((warp & 3) == 0) {
                // Sylvester FWHT of so in one warp: element VPL*lane + k
                constexpr int VPL = D / 32;
                float v[VPL];
#pragma unroll
                for (int k = 0; k < VPL; ++k) v[k] = so[VPL * lane + k];
#pragma unroll
                for (int h = 1; h < VPL; h <<= 1)
#pragma unroll
                    for (int k = 0; k < VPL; ++k)
                        if ((k & h) == 0) {
                            const float x0 = v[k], x1 = v[k + h];
                            v[k] = x0 + x1;
                            v[k + h] = x0 - x1;
                        }
#pragma unroll
                for (int hl = 1; hl < 32; hl <<= 1)
#pragma unroll
                    for (int k = 0; k < VPL; ++k) {
                        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[k], hl);
                        v[k] = (lane & hl) ? o - v[k] : v[k] + o;
                    }
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    const int j = VPL * lane + k;  // coordinate j sits in column (j&~31) + 2(j&15) + ((j>>4)&1)
                    ho[(j & ~31) + ((j & 15) << 1) + ((j >> 4) & 1)] = v[k];
                }
            }
            named_bar_sync(bar_id, 128);
        }
        const bool okh = mbar_wait(&hbar[wg], hpar, a.status);
        hpar ^= 1u;
        if (named_bar_or(bar_id, 128, !okh)) break;
        if (r == 0) issue_tile(i + NS);  // the stage has been read
        tc_fence_after();

        // -ho for the pair idx of the rotated vector (column order), read as the
        // 16-byte chunk holding pairs idx & ~1 and idx | 1 (one load serves both)
        auto ho_neg = [&](int idx) {
            const float4 hq = reinterpret_cast<const float4*>(ho)[idx >> 1];
            return (idx & 1) ? make_float2(-hq.z, -hq.w) : make_float2(-hq.x, -hq.y);
        };
        float nrm, rr;
        uint32_t planes[B][kWpp];
        if constexpr (C::kNMat == 1) {
            // ---- pass 1: ||y||^2 = D ||x||^2 (the next chunk loads while one is summed) ----
            constexpr int NC = D / 32;
            uint32_t ybuf[2][32];
            float2 acc2 = make_float2(0.f, 0.f);
            tmem_ld32(tl, ybuf[0]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                if (c + 1 < NC) tmem_ld32(tl + 32 * (c + 1), ybuf[(c + 1) & 1]);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    float2 y = make_float2(u2f(ybuf[c & 1][2 * k]), u2f(ybuf[c & 1][2 * k + 1]));
                    if constexpr (NSN) y = __ffma2_rn(y, make_float2(sc, sc), ho_neg(16 * c + k));  // H D w
                    acc2 = __ffma2_rn(y, y, acc2);
                }
                if (c + 1 < NC) tmem_wait_ld();
            }
            const float ssx = (acc2.x + acc2.y) * (1.0f / D);
            nrm = sqrtf(ssx);  // ||x||, or ||w|| for NSN
            if (!NSN) flag_norm(ssx, nrm, a.status);
            const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
            // ---- pass 2: codes, residual (fp16 into columns [16c, 16c + 16)) ----
            // Group c + 1 loads while group c is coded; the residual of group c
            // goes to columns that groups 0 .. c/2 occupied, all read already.
            float2 rr2 = make_float2(0.f, 0.f);
            const VecTab<B> vt(ctab, nrm, inv);
            tmem_ld32(tl, ybuf[0]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                if (c + 1 < NC) tmem_ld32(tl + 32 * (c + 1), ybuf[(c + 1) & 1]);
                float2 v[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    v[k] = make_float2(u2f(ybuf[c & 1][2 * k]), u2f(ybuf[c & 1][2 * k + 1]));
                    if constexpr (NSN) v[k] = __ffma2_rn(v[k], make_float2(sc, sc), ho_neg(16 * c + k));
                }
                uint32_t hres[16], w[B];
                code_group<B>(v, ctab, vt, hres, w, rr2);
#pragma unroll
                for (int p = 0; p < B; ++p) planes[p][c] = w[p];
                // Stored without QJL too (except behind the NSN front end): consuming
                // the residual group by group keeps the register allocation within
                // the 128 registers of a thread.
                if (!NSN) tmem_st16(tl + 16 * c, hres);
                if (c + 1 < NC) tmem_wait_ld();
            }
            rr = rr2.x + rr2.y;
        } else {
            // ---- d = 256: columns [0, 128) hold P, [128, 256) Q; group c < 4 of
            // the rotated vector is P_c + Q_c, group 4 + c is P_c - Q_c ----
            const float2 m1 = make_float2(-1.f, -1.f);
            const float2 sc2 = make_float2(sc, sc);
            // y of group (c, half) from the loaded P and Q words, pair k
            auto ypair = [&](const uint32_t(&pw)[32], const uint32_t(&qw)[32], int c, int half, int k) {
                const float2 pv = make_float2(u2f(pw[2 * k]), u2f(pw[2 * k + 1]));
                const float2 qv = make_float2(u2f(qw[2 * k]), u2f(qw[2 * k + 1]));
                float2 y = half ? __ffma2_rn(qv, m1, pv) : __fadd2_rn(pv, qv);
                if constexpr (NSN) y = __ffma2_rn(y, sc2, ho_neg(16 * (4 * half + c) + k));  // H D w
                return y;
            };
            // One buffer: both halves of group c are formed from P_c and Q_c,
            // then P_{c+1} and Q_{c+1} load into the same registers while
            // group c is summed or coded.
            // (pin2 keeps the formed values from being computed after the next
            // load, which would keep the old P and Q words live beside it)
            auto pin2 = [](float2& v) { asm volatile("" : "+f"(v.x), "+f"(v.y)); };
            uint32_t pb[32], qb[32];
            // ---- pass 1: ||y||^2 (without the NSN shift, 2 (||P||^2 + ||Q||^2)) ----
            float2 acc2 = make_float2(0.f, 0.f);
            tmem_ld32(tl, pb);
            tmem_ld32(tl + 128, qb);
            tmem_wait_ld();
            if constexpr (!NSN) {
                float2 accq = make_float2(0.f, 0.f);
                // P_{c+1} loads while Q_c is summed
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float2 pv = make_float2(u2f(pb[2 * k]), u2f(pb[2 * k + 1]));
                        acc2 = __ffma2_rn(pv, pv, acc2);
                    }
                    pin2(acc2);
                    if (c + 1 < 4) tmem_ld32(tl + 32 * (c + 1), pb);
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float2 qv = make_float2(u2f(qb[2 * k]), u2f(qb[2 * k + 1]));
                        accq = __ffma2_rn(qv, qv, accq);
                    }
                    pin2(accq);
                    if (c + 1 < 4) {
                        tmem_ld32(tl + 128 + 32 * (c + 1), qb);
                        tmem_wait_ld();
                    }
                }
                acc2 = __fadd2_rn(acc2, accq);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float2 yt[16], yb[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        yt[k] = ypair(pb, qb, c, 0, k);
                        yb[k] = ypair(pb, qb, c, 1, k);
                        pin2(yt[k]);
                        pin2(yb[k]);
                    }
                    if (c + 1 < 4) {
                        tmem_ld32(tl + 32 * (c + 1), pb);
                        tmem_ld32(tl + 128 + 32 * (c + 1), qb);
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        acc2 = __ffma2_rn(yt[k], yt[k], acc2);
                        acc2 = __ffma2_rn(yb[k], yb[k], acc2);
                    }
                    if (c + 1 < 4) tmem_wait_ld();
                }
            }
            const float ssx = (acc2.x + acc2.y) * ((NSN ? 1.0f : 2.0f) / D);
            nrm = sqrtf(ssx);  // ||x||, or ||w|| for NSN
            if (!NSN) flag_norm(ssx, nrm, a.status);
            const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
            // ---- pass 2: codes of both halves of each group (no QJL: the residual is only summed) ----
            float2 rr2 = make_float2(0.f, 0.f);
            const VecTab<B> vt(ctab, nrm, inv);
            tmem_ld32(tl, pb);
            tmem_ld32(tl + 128, qb);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float2 yt[16], yb[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    yt[k] = ypair(pb, qb, c, 0, k);
                    yb[k] = ypair(pb, qb, c, 1, k);
                    pin2(yt[k]);
                    pin2(yb[k]);
                }
                if (c + 1 < 4) {
                    tmem_ld32(tl + 32 * (c + 1), pb);
                    tmem_ld32(tl + 128 + 32 * (c + 1), qb);
                }
                uint32_t hres[16], w[B];
                code_group<B>(yt, ctab, vt, hres, w, rr2);
#pragma unroll
                for (int p = 0; p < B; ++p) planes[p][c] = w[p];
                code_group<B>(yb, ctab, vt, hres, w, rr2);
#pragma unroll
                for (int p = 0; p < B; ++p) planes[p][4 + c] = w[p];
                if (c + 1 < 4) tmem_wait_ld();
            }
            rr = rr2.x + rr2.y;
        }
        const uint32_t zmask = nrm > 0.f ? 0xFFFFFFFFu : 0u;
        const int64_t vidx = tile * kTileRows + r;
        const bool valid = vidx < n_s;
        if (layout_s == 0) {
            if (valid) {
                uint32_t* cp = codes_s + vidx * (B * kWpp);
#pragma unroll
                for (int p = 0; p < B; ++p) store_words<kWpp>(cp + p * kWpp, planes[p], zmask);
            }
        } else {
            const int64_t blk = tile * 4 + (warp & 3);
            const uint32_t m = valid ? zmask : 0u;
#pragma unroll
            for (int p = 0; p < B; ++p)
                store_block32_t<kWpp>(codes_s + (blk * B + p) * D, planes[p], m, lane, blk * 32 < n_s);
        }
        if (valid) {
            const float g = nrm > 0.f ? sqrtf(rr) : 0.f;
            if constexpr (DQ) reinterpret_cast<__half*>(norms_s)[vidx] = __float2half_rn(nrm);  // ||w|| only
            else
                norms_s[vidx] = NSN ? __halves2half2(__float2half_rn(nx), __float2half_rn(nrm))
                                    : __halves2half2(__float2half_rn(nrm), __float2half_rn(g));
        }

        if (QJL) {
            // ---- QJL: U = R S_h^T per 64-row half of S, in columns [64, 128) ----
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(bar_id, 128);
            uint32_t qw[kWpp];
            bool failed = false;
#pragma unroll
            for (int h = 0; h < D / C::kQN; ++h) {
                if (r == 0) {
                    tc_fence_after();
                    const uint32_t ss0 = smem_u32(sS);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t boff = (ks / 4) * (D * 128) + h * (C::kQN * 128) + (ks % 4) * 32;
                        mma_f16_ts(tcol + 64, tcol + ks * 8, smem_desc_sw128(ss0 + boff), kIdescQ,
                                   ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&qbar[wg]);
                }
                const bool okq = mbar_wait(&qbar[wg], qpar, a.status);
                qpar ^= 1u;
                if (named_bar_or(bar_id, 128, !okq)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                uint32_t u0[32], u1[32];
                tmem_ld32(tl + 64, u0);
                tmem_ld32(tl + 96, u1);
                tmem_wait_ld();
                qw[2 * h] = sign_word(u0);
                qw[2 * h + 1] = sign_word(u1);
                tc_fence_before();
                if (h + 1 < D / C::kQN) named_bar_sync(bar_id, 128);  // the next half reuses the columns
            }
            if (failed) break;
            if (layout_s == 0) {
                if (valid) store_words<kWpp>(qjl_s + vidx * kWpp, qw, zmask);
            } else {
                const int64_t blk = tile * 4 + (warp & 3);
                store_block32_t<kWpp>(qjl_s + blk * D, qw, valid ? zmask : 0u, lane, blk * 32 < n_s);
            }
        }
        // The next rotation MMA rewrites this warpgroup's columns; the barrier
        // at the top of the next iteration orders it after these accesses.
        tc_fence_before();
    }

    __syncthreads();
    if (tid == 0) {
        // Loads issued but never consumed (only after a wait gave up).
        for (int s = 0; s < NS; ++s)
            if (iss[s] > con[s]) mbar_wait(&full[s], con[s] & 1u, a.status);
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int B, bool QJL, int DT, bool NSN = false, bool DQ = false>
cudaError_t launch_quantize_tc(const CUtensorMap& map, const CUtensorMap& map1, const QuantArgs& a, int num_sms,
                               cudaStream_t s) {
    using C = TcCfg<D, QJL, NSN>;
    auto kern = quantize_tc_kernel<D, B, QJL, DT, NSN, DQ>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t grid = a.ntiles < num_sms ? a.ntiles : num_sms;
    if (grid <= 0) return cudaSuccess;
    // Programmatic dependent launch: this grid may be scheduled while the
    // previous one drains; the kernel waits for it before touching memory.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, map, map1, a);
}

}  // namespace kvq
