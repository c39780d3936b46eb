// quantize_tc.cuh -- the quantize kernel (and its NSN front end) with the
// rotation on the tensor cores, for 16-bit input and d <= 128.
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
    static constexpr int kMatBytes = D * D * 2;            // H D or S, 16-bit, K-major, swizzled
    static constexpr int kWG = 4;
    static constexpr int kThreads = 128 * kWG;
    static constexpr int kAuxBytes = NSN ? 12288 : 1024;  // NSN: per-warpgroup scale, partial means, mean, rotated mean
    static constexpr int kBudget = 225 * 1024;
    static constexpr int kStagesRaw = (kBudget - kMatBytes - (QJL ? kMatBytes : 0) - kAuxBytes) / kTileBytes;
    // Tile i goes to warpgroup i % 4 and stage i % kStages; with kStages a
    // multiple of 4 every stage belongs to one warpgroup, which consumes its
    // phases strictly in order (a parity wait can never see a stale phase).
    static constexpr int kStages = (kStagesRaw > 8 ? 8 : kStagesRaw) / kWG * kWG;
    static constexpr int kSmemBytes = 1024 + kStages * kTileBytes + kMatBytes + (QJL ? kMatBytes : 0) + kAuxBytes;
    static constexpr int kQN = 64;                          // rows of S per QJL MMA
    static_assert(D == 64 || D == 128, "tensor-core rotation: d in {64, 128}");
    static_assert(kStages >= kWG, "one stage per warpgroup at least");
};

// Sign word of 32 accumulator values: bit i = [u_i >= 0].
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&u)[32]) {
    uint32_t b[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 7; i >= 0; --i)
#pragma unroll
        for (int q = 0; q < 4; ++q) b[q] = __funnelshift_l(u[8 * q + i], b[q], 1);
    return ~(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24));
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

template <int D, int B, bool QJL, int DT, bool NSN = false>
__global__ void __launch_bounds__(512, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap map, const __grid_constant__ CUtensorMap map1,
                       const __grid_constant__ QuantArgs a) {
    static_assert(!(NSN && QJL), "NSN front end: no QJL");
    using C = TcCfg<D, QJL, NSN>;
    constexpr int NS = C::kStages;
    constexpr int kWpp = D / 32;
    constexpr uint32_t kIdescH = idesc_16bit_f32(kTileRows, D, DT == DT_BF16);
    constexpr uint32_t kIdescQ = idesc_16bit_f32(kTileRows, C::kQN, false);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage0 = smem;
    uint8_t* sHD = smem + NS * C::kTileBytes;
    uint8_t* sS = sHD + C::kMatBytes;
    uint8_t* aux = sS + (QJL ? C::kMatBytes : 0);
    uint64_t* full = reinterpret_cast<uint64_t*>(aux);    // [8]
    uint64_t* hbar = full + 8;                              // [4] rotation MMA done
    uint64_t* qbar = hbar + 4;                              // [4] QJL MMA done
    uint32_t* iss = reinterpret_cast<uint32_t*>(qbar + 4);  // [8] loads issued per stage
    uint32_t* con = iss + 8;                                // [8] loads consumed per stage
    uint32_t* tmem_slot = con + 8;
    float* nsn_aux = reinterpret_cast<float*>(aux + 1024);  // NSN: [4 warpgroups][640]

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
    // H D as the B operand (row n = output coordinate, K = input coordinate):
    // entry (n, k) = (-1)^popcount(n & k) delta_k.  K-chunk kc (64 entries)
    // of row n at sHD + kc*D*128 + n*128, 16-byte chunk c at c ^ (n & 7).
    {
        const uint32_t one = (DT == DT_BF16) ? 0x3F80u : 0x3C00u;
        for (int e = tid; e < D * D / 8; e += C::kThreads) {
            const int n = e / (D / 8), cc = e % (D / 8);
            const int kc = cc / 8, c16 = cc % 8;
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int k = 8 * cc + 2 * q;
                const uint32_t ps = a.pair_sign[k >> 1];
                const uint32_t s0 = ((__popc(n & k) & 1u) << 15) ^ (ps & 0x8000u);
                const uint32_t s1 = ((__popc(n & (k + 1)) & 1u) << 15) ^ ((ps >> 16) & 0x8000u);
                w4[q] = (one | s0) | ((one | s1) << 16);
            }
            *reinterpret_cast<uint4*>(sHD + kc * (D * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
    if (QJL) {
        // S is written once at handle creation, before any launch.
        const uint4* gS = reinterpret_cast<const uint4*>(a.S);
        for (int e = tid; e < D * D / 8; e += C::kThreads) {
            const int n = e / (D / 8), cc = e % (D / 8);
            const int kc = cc / 8, c16 = cc % 8;
            *reinterpret_cast<uint4*>(sS + kc * (D * 128) + n * 128 + ((c16 ^ (n & 7)) << 4)) = gS[e];
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
    const uint32_t tcol = tmem + static_cast<uint32_t>(wg * 128);  // this warpgroup's 128 columns
    const uint32_t tl = tcol + lane_base;                            // ... at this thread's lane
    uint32_t hpar = 0, qpar = 0;

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
            // ---- rotation: Y = X (H D)^T into columns [0, D) ----
            tc_fence_after();
            const uint32_t xs = smem_u32(stage0 + st * C::kTileBytes);
            const uint32_t hs = smem_u32(sHD);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t aoff = (ks / 4) * C::kBoxBytes + (ks % 4) * 32;
                const uint32_t boff = (ks / 4) * (D * 128) + (ks % 4) * 32;
                mma_f16_ss(tcol, smem_desc_sw128(xs + aoff), smem_desc_sw128(hs + boff), kIdescH, ks > 0 ? 1u : 0u);
            }
            mma_commit(&hbar[wg]);
        }
        // NSN front end on the tile (= one block of 128 tokens of one head):
        // sc = sqrt(D)/||x||, block mean o of u = sc x per channel, fp16(o),
        // and ho = H (delta .* fp16(o)), so that H D w = sc y - ho.
        float nx = 0.f, sc = 0.f;
        float* xch = nsn_aux + wg * 640;  // [128] sc per token
        float* so = xch + 128;            // [D] delta .* fp16(o)
        float* ho = xch + 256;            // [D] H (delta .* fp16(o))
        float2* opart = reinterpret_cast<float2*>(xch + 384);  // [128 / (D/2)][D/2] partial channel sums
        if constexpr (NSN) {
            const uint8_t* sp = stage0 + st * C::kTileBytes;
            const float ssx0 = stage_row_sumsq<D, DT>(sp, r);
            nx = sqrtf(ssx0);
            flag_norm(ssx0, nx, a.status);
            sc = nx > 0.f ? sqrtf(static_cast<float>(D)) / nx : 0.f;
            xch[r] = sc;
            named_bar_sync(bar_id, 128);
            {
                // thread r: channel pair p, tokens of group q (fp32x2 sums)
                constexpr int P = D / 2, Q = kTileRows / P, TPQ = kTileRows / Q;
                const int p = r % P, q = r / P;
                const int j0 = 2 * p;
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
                for (int t = q * TPQ; t < (q + 1) * TPQ; ++t) {
                    const uint32_t wd = *reinterpret_cast<const uint32_t*>(
                        sp + (j0 / 64) * 16384 + t * 128 + ((((j0 % 64) / 8) ^ (t & 7)) << 4) + (j0 % 8) * 2);
                    const float2 xv = (DT == DT_BF16) ? make_float2(u2f(wd << 16), u2f(wd & 0xFFFF0000u))
                                                      : __half22float2(*reinterpret_cast<const __half2*>(&wd));
                    const float sct = xch[t];
                    acc = __ffma2_rn(xv, make_float2(sct, sct), acc);
                }
                opart[q * P + p] = acc;
            }
            named_bar_sync(bar_id, 128);
            if (r < D) {
                constexpr int P = D / 2, Q = kTileRows / P;
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const float2 pq = opart[q * P + r / 2];
                    acc += (r & 1) ? pq.y : pq.x;
                }
                const __half o16 = __float2half_rn(acc * (1.0f / kTileRows));
                if (tile * kTileRows < n_s) a.block_mean[tile * D + r] = o16;
                const uint32_t ps = a.pair_sign[r >> 1];
                const bool neg = ((ps >> ((r & 1) ? 31 : 15)) & 1u) != 0;
                so[r] = neg ? -__half2float(o16) : __half2float(o16);
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
                for (int k = 0; k < VPL; ++k) ho[VPL * lane + k] = v[k];
            }
            named_bar_sync(bar_id, 128);
        }
        const bool okh = mbar_wait(&hbar[wg], hpar, a.status);
        hpar ^= 1u;
        if (named_bar_or(bar_id, 128, !okh)) break;
        if (r == 0) issue_tile(i + NS);  // the stage has been read
        tc_fence_after();

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
                if constexpr (NSN) {
                    const float2 h2 = reinterpret_cast<const float2*>(ho)[16 * c + k];
                    y = __ffma2_rn(y, make_float2(sc, sc), make_float2(-h2.x, -h2.y));  // H D w
                }
                acc2 = __ffma2_rn(y, y, acc2);
            }
            if (c + 1 < NC) tmem_wait_ld();
        }
        const float ssx = (acc2.x + acc2.y) * (1.0f / D);
        const float nrm = sqrtf(ssx);  // ||x||, or ||w|| for NSN
        if (!NSN) flag_norm(ssx, nrm, a.status);
        const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;

        // ---- pass 2: codes, residual (fp16 into columns [16c, 16c + 16)) ----
        // Chunk c + 1 loads while chunk c is coded; the residual of chunk c
        // goes to columns that chunks 0 .. c/2 occupied, all read already.
        uint32_t planes[B][kWpp];
        float rr = 0.f;
        tmem_ld32(tl, ybuf[0]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            if (c + 1 < NC) tmem_ld32(tl + 32 * (c + 1), ybuf[(c + 1) & 1]);
            float2 v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                v[k] = make_float2(u2f(ybuf[c & 1][2 * k]), u2f(ybuf[c & 1][2 * k + 1]));
                if constexpr (NSN) {
                    const float2 h2 = reinterpret_cast<const float2*>(ho)[16 * c + k];
                    v[k] = __ffma2_rn(v[k], make_float2(sc, sc), make_float2(-h2.x, -h2.y));
                }
            }
            uint32_t pl[B][1];
            rr += codes_and_residual<32, B>(v, inv, a, pl);
#pragma unroll
            for (int p = 0; p < B; ++p) planes[p][c] = pl[p][0];
            if (QJL) {
                uint32_t hi[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const __half2 hh = __float22half2_rn(v[k]);
                    hi[k] = *reinterpret_cast<const uint32_t*>(&hh);
                }
                tmem_st16(tl + 16 * c, hi);
            }
            if (c + 1 < NC) tmem_wait_ld();
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
                store_block32<kWpp>(codes_s + (blk * B + p) * D, planes[p], m, lane, blk * 32 < n_s);
        }
        if (valid) {
            const float g = nrm > 0.f ? sqrtf(rr) : 0.f;
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
                store_block32<kWpp>(qjl_s + blk * D, qw, valid ? zmask : 0u, lane, blk * 32 < n_s);
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

template <int D, int B, bool QJL, int DT, bool NSN = false>
cudaError_t launch_quantize_tc(const CUtensorMap& map, const CUtensorMap& map1, const QuantArgs& a, int num_sms,
                               cudaStream_t s) {
    using C = TcCfg<D, QJL, NSN>;
    auto kern = quantize_tc_kernel<D, B, QJL, DT, NSN>;
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
