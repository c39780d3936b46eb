// decode.cu -- decode attention straight from the packed cache.
//
// Method (TurboQuant blog, "Como Implementar": the query is rotated once and
// the logits come from the stored indices; PolarQuant section 2: the
// dequantisation H^T/d, the centroid lookup and the stored norm, here moved
// to the query side and to one final inverse rotation):
//   q' = H (delta .* q), p = S q'                              (qproj_kernel)
//   l_t = scale (n_t/d) (<q', c[code_t]> + sqrt(pi/2)/m gamma_t <p, sgn_t>)
//   per split of the context: running max M, sum L, A = sum w n c[vcode],
//   B = sum w n gamma sgn_v                                   (decode_split_kernel)
//   merge the splits exactly, out = delta .* H (A + sqrt(pi/2)/m S^T B) / (d L)
//                                                              (decode_combine_kernel)
// Three launches on one stream (a fourth, decode_window_kernel, for a
// residual window); the split partials live in the caller's workspace.  No
// kernel waits on another CTA.  This file holds the CUDA-core path (4-bit
// codebooks, and 3-bit at d = 256), the combine and window kernels shared
// with the tensor-core path of decode_mma.cu, and the split plan.
#include <cfloat>
#include <mutex>

#include <type_traits>

#include "kvq_internal.h"
#include "sm100.cuh"

namespace kvq {

// Fixed device scratch used by kvq_decode_attend_noalloc in place of a
// caller-provided workspace.  A file-scope __device__ array: every GPU that
// loads this library holds kNoAllocScratchBytes of it until the process
// exits.  Host code must not use the symbol itself as a device address; the
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(int device, void** ptr) {
    // Looked up once per device, with that device current (the caller makes
    // sure it is), and cached; later calls only read the cache.
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[device] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[device] = p;
    }
    *ptr = addr[device];
    return cudaSuccess;
}

namespace {

constexpr int kDecThreads = 256;
constexpr int kTokTile = 256;  // tokens per split granule
constexpr float kSqrtHalfPi = 1.2533141373155002512f;  // sqrt(pi/2)

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i) {
    if (DT == 0) return reinterpret_cast<const float*>(p)[i];
    if (DT == 1) return __half2float(reinterpret_cast<const __half*>(p)[i]);
    const uint16_t u = reinterpret_cast<const uint16_t*>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

__device__ __forceinline__ float sign_of(const uint32_t* pair_sign, int j) {
    return ((pair_sign[j >> 1] >> ((j & 1) ? 31 : 15)) & 1u) ? -1.f : 1.f;
}

// In-place FWHT of D floats in shared memory by the whole block.
template <int D>
__device__ __forceinline__ void fwht_smem(float* s) {
    for (int h = 1; h < D; h <<= 1) {
        for (int p = threadIdx.x; p < D / 2; p += blockDim.x) {
            const int i = (p / h) * 2 * h + (p % h);
            const float x = s[i], y = s[i + h];
            s[i] = x + y;
            s[i + h] = x - y;
        }
        __syncthreads();
    }
}

// q' = H (delta .* q) and p = S q' for one (batch, query head) per block.
template <int D, int DT, bool QJL>
__global__ void __launch_bounds__(kDecThreads) qproj_kernel(const __grid_constant__ DecodeArgs a) {
    __shared__ float sq[D];
    const int64_t bh = blockIdx.x;
    for (int j = threadIdx.x; j < D; j += blockDim.x)
        sq[j] = sign_of(a.pair_sign, j) * load_elem<DT>(a.q, bh * D + j);
    __syncthreads();
    fwht_smem<D>(sq);
    for (int j = threadIdx.x; j < D; j += blockDim.x) a.qrot[bh * D + j] = sq[j];
    if (QJL) {
        // row i of S by 16-byte loads, eight in flight at a time
        for (int i = threadIdx.x; i < D; i += blockDim.x) {
            const uint4* Si = reinterpret_cast<const uint4*>(a.S + static_cast<int64_t>(i) * D);
            float acc = 0.f;
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
                        acc = fmaf(sv.y, sq[j + 1], fmaf(sv.x, sq[j], acc));
                    }
                }
            }
            a.qproj[bh * D + i] = acc;
        }
    }
}

template <int B>
__device__ __forceinline__ int code_at(const uint32_t* planes, int words_per_plane, int j) {
    int code = 0;
#pragma unroll
    for (int p = 0; p < B; ++p) code |= static_cast<int>((planes[p * words_per_plane + (j >> 5)] >> (j & 31)) & 1u) << p;
    return code;
}

// One (split, kv head, batch) per block: tokens [split*chunk, (split+1)*chunk).
// NSN (no QJL): caches written by the NSN front end, fp16 block means per 128
// tokens (NSNQuant sections 1 and 4): the logit is scale ||x||/sqrt(d)
// (||w||/d <q', c[code]> + <q, o_blk>), the code weights are e ||x|| ||w|| / sqrt(d)
// and the block means enter the partial's second vector with e ||x|| / sqrt(d).
// DQ (with NSN): the norms hold fp16 ||w|| per token and the block means are
// side records (4-bit codes of ||x|| and of the means, NSNQuant section 3):
// ||x|| reads as n1 = q nstep and the mean as o_hat = lo + step q.
template <int D, int B, bool QJL, int G, bool NSN = false, bool DQ = false>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeArgs a) {
    static_assert(!(NSN && QJL), "NSN caches carry no QJL sketch");
    static_assert(!DQ || NSN, "double-quantized side data belong to NSN caches");
    constexpr int RB = (8 + D / 2 + 64 + 15) / 16 * 16;  // DQ: bytes of one side record
    constexpr int M = D;                 // QJL rows
    constexpr int WP = D / 32;           // words per plane
    constexpr int KW = B * WP;           // code words per vector
    constexpr int QW = QJL ? M / 32 : 0; // sign words per vector
    constexpr int PART = 2 + D + M;
    constexpr int TT = (D == 256) ? 128 : 256;  // tokens per tile (one per thread of phase A)
    const int split = blockIdx.x, hk = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x;

    __shared__ float sqr[G][D];
    __shared__ float spq[G][QJL ? M : 1];
    __shared__ float scb[1 << B];
    __shared__ float sw[G][TT];                  // softmax weights of the tile
    __shared__ uint32_t svc[TT / 32][B][D];      // value code planes of the tile (block-32 layout)
    __shared__ uint32_t svq[TT / 32][QJL ? M : 1];
    __shared__ float svn[TT], svg[TT];
    __shared__ float sred[G][kDecThreads / 32];
    __shared__ float smax[G], salpha[G], ssum[G];
    constexpr int NBT = TT / 128;                      // NSN blocks per tile
    __shared__ float sq0[NSN ? G : 1][NSN ? D : 1];    // NSN: the query in the original domain
    __shared__ float sqo[G][NBT];                      // NSN: scale/sqrt(d) <q, o_blk> of the tile's blocks
    __shared__ float sbeta[G][NBT];                    // NSN: sum of e ||x|| / sqrt(d) per block of the tile
    const float inv_sqrt_d = rsqrtf(static_cast<float>(D));

    const int64_t T = min(static_cast<int64_t>(max(a.seq_len[bi], 0)), a.max_T);
    const int64_t t0 = static_cast<int64_t>(split) * a.chunk;
    const int64_t t1e = min(t0 + a.chunk, a.max_T);       // range this split owns (logit output)
    const int64_t t1 = min(t1e, T);                        // tokens that exist
    const int64_t stream = static_cast<int64_t>(bi) * a.hkv + hk;
    const int64_t qh0 = static_cast<int64_t>(bi) * a.hq + static_cast<int64_t>(hk) * G;

    for (int e = tid; e < G * D; e += blockDim.x) sqr[e / D][e % D] = a.qrot[(qh0 + e / D) * D + e % D];
    if (QJL)
        for (int e = tid; e < G * M; e += blockDim.x) spq[e / M][e % M] = a.qproj[(qh0 + e / M) * M + e % M];
    if (tid < (1 << B)) scb[tid] = a.centroid[tid];
    if constexpr (NSN) {
        for (int e = tid; e < G * D; e += blockDim.x) {
            const int64_t i = (qh0 + e / D) * D + e % D;
            const uint16_t u = reinterpret_cast<const uint16_t*>(a.q)[a.qdtype == 0 ? 0 : i];
            sq0[e / D][e % D] = a.qdtype == 0 ? reinterpret_cast<const float*>(a.q)[i]
                                : a.qdtype == 1 ? __half2float(__ushort_as_half(u))
                                                : __uint_as_float(static_cast<uint32_t>(u) << 16);
        }
    }
    if (tid < G) {
        smax[tid] = -INFINITY;
        ssum[tid] = 0.f;
    }
    // value-side accumulators: thread role A (coordinate tid < D) and B (row tid - D < M)
    float accA[G], accB[G], accA2[G], accB2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) accA[g] = accB[g] = accA2[g] = accB2[g] = 0.f;
    __syncthreads();

    const uint32_t* kc = a.kcodes + stream * a.kcap * KW;
    const uint32_t* kq = QJL ? a.kqjl + stream * a.kcap * QW : nullptr;
    const __half2* kn = a.knorms + stream * a.kcap;
    // values: block-32 layout, capacity a multiple of 32
    const uint32_t* vc = a.vcodes + stream * (a.vcap / 32) * B * D;
    const uint32_t* vq = QJL ? a.vqjl + stream * (a.vcap / 32) * M : nullptr;
    const __half2* vn = a.vnorms + stream * a.vcap;
    const float kappa = kSqrtHalfPi / M;
    const __half* kmean = (NSN && !DQ) ? a.kmean + stream * (a.kcap / 128) * D : nullptr;
    const __half* vmean = (NSN && !DQ) ? a.vmean + stream * (a.vcap / 128) * D : nullptr;
    const uint8_t* krec = DQ ? reinterpret_cast<const uint8_t*>(a.kmean) + stream * (a.kcap / 128) * RB : nullptr;
    const uint8_t* vrec = DQ ? reinterpret_cast<const uint8_t*>(a.vmean) + stream * (a.vcap / 128) * RB : nullptr;
    auto f16at = [](const uint8_t* p) { return __half2float(*reinterpret_cast<const __half*>(p)); };
    auto nib = [](const uint8_t* p, int i) { return static_cast<float>((p[i >> 1] >> ((i & 1) * 4)) & 15); };
    // block mean of channel j (fp16 as stored, or o_hat from the record) and the stored norms of token t
    auto kmean_at = [&](int64_t blk, int j) {
        if constexpr (DQ) {
            const uint8_t* r = krec + blk * RB;
            return fmaf(f16at(r + 2), nib(r + 8, j), f16at(r));
        } else {
            return __half2float(kmean[blk * D + j]);
        }
    };
    auto vmean_at = [&](int64_t blk, int j) {
        if constexpr (DQ) {
            const uint8_t* r = vrec + blk * RB;
            return fmaf(f16at(r + 2), nib(r + 8, j), f16at(r));
        } else {
            return __half2float(vmean[blk * D + j]);
        }
    };
    // DQ norms: one fp16 ||w|| per token (the stream's base in fp16 units)
    const __half* knh = reinterpret_cast<const __half*>(a.knorms) + stream * a.kcap;
    const __half* vnh = reinterpret_cast<const __half*>(a.vnorms) + stream * a.vcap;
    auto norms_at = [&](bool key, int64_t tt) -> float2 {
        if constexpr (DQ) {
            const uint8_t* r = (key ? krec : vrec) + (tt >> 7) * RB;
            const float n1 = nib(r + 8 + D / 2, static_cast<int>(tt & 127)) * f16at(r + 4);
            return make_float2(n1, __half2float((key ? knh : vnh)[tt]));
        } else {
            return __half22float2((key ? kn : vn)[tt]);
        }
    };

    for (int64_t tb = t0; tb < t1e; tb += TT) {
        if constexpr (NSN) {
            // scale/sqrt(d) <q_g, o_blk> for the tile's blocks (tb is a multiple of 128); a
            // block past the cache's tokens gives a value no valid token uses
            const int warp = tid >> 5, lane = tid & 31;
            for (int pr = warp; pr < G * NBT; pr += kDecThreads / 32) {
                const int g = pr / NBT, bq = pr % NBT;
                const int64_t blk = tb / 128 + bq;
                float acc = 0.f;
                if (blk * 128 < t1)
                    for (int j = lane; j < D; j += 32) acc = fmaf(sq0[g][j], kmean_at(blk, j), acc);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (lane == 0) sqo[g][bq] = acc * a.scale * inv_sqrt_d;
            }
            __syncthreads();
        }
        // ---- phase A: logits, one token per thread ----
        const int64_t t = tb + tid;
        const bool mine = tid < TT;
        float l[G];
        if (mine && t < t1) {
            uint32_t cw[KW];
#pragma unroll
            for (int w = 0; w < KW; ++w) cw[w] = kc[t * KW + w];
            float acc[G], accq[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = accq[g] = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) {
                const float c = scb[code_at<B>(cw, WP, j)];
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = fmaf(sqr[g][j], c, acc[g]);
            }
            const float2 nk = norms_at(true, t);
            if (QJL) {
                uint32_t qw[QJL ? QW : 1];
#pragma unroll
                for (int w = 0; w < QW; ++w) qw[w] = kq[t * QW + w];
#pragma unroll
                for (int i = 0; i < M; ++i) {
                    const float s = ((qw[i >> 5] >> (i & 31)) & 1u) ? 1.f : -1.f;
#pragma unroll
                    for (int g = 0; g < G; ++g) accq[g] = fmaf(spq[g][i], s, accq[g]);
                }
            }
            if constexpr (NSN) {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    l[g] = nk.x * fmaf(a.scale * inv_sqrt_d * (nk.y / D), acc[g], sqo[g][tid >> 7]);
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    l[g] = a.scale * (nk.x / D) * (acc[g] + (QJL ? kappa * nk.y * accq[g] : 0.f));
            }
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g) l[g] = -INFINITY;
        }
        if (a.logits != nullptr && mine && t < t1e) {
#pragma unroll
            for (int g = 0; g < G; ++g) a.logits[(qh0 + g) * a.logits_ld + t] = l[g];
        }
        // stage the value bit planes (blocks of 32 tokens) and norms of this tile
        {
            const int64_t blk0 = tb / 32;
            const int nblk = static_cast<int>(min(static_cast<int64_t>(TT / 32), (t1 - tb + 31) / 32 > 0 ? (t1 - tb + 31) / 32 : 0));
            for (int e = tid; e < nblk * B * D; e += kDecThreads)
                (&svc[0][0][0])[e] = vc[blk0 * B * D + e];
            if (QJL)
                for (int e = tid; e < nblk * M; e += kDecThreads) (&svq[0][0])[e] = vq[blk0 * M + e];
        }
        if (mine && t < t1) {
            // NSN: the code weight factor ||x|| ||w|| / sqrt(d) and the block-mean factor ||x|| / sqrt(d)
            const float2 nv = norms_at(false, t);
            svn[tid] = NSN ? nv.x * nv.y * inv_sqrt_d : nv.x;
            svg[tid] = NSN ? nv.x * inv_sqrt_d : nv.y;
        }
        // ---- phase B: tile max, running max, weights ----
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float mx = l[g];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if ((tid & 31) == 0) sred[g][tid >> 5] = mx;
        }
        __syncthreads();
        if (tid < G) {
            float mx = sred[tid][0];
            for (int k = 1; k < kDecThreads / 32; ++k) mx = fmaxf(mx, sred[tid][k]);
            const float mold = smax[tid];
            const float mnew = fmaxf(mold, mx);
            salpha[tid] = (mnew == -INFINITY) ? 1.f : __expf(mold - mnew);
            smax[tid] = mnew;
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mnew = smax[g];
            const float wgt = (l[g] == -INFINITY) ? 0.f : __expf(l[g] - mnew);
            if (mine) sw[g][tid] = wgt;
            float s = wgt;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if ((tid & 31) == 0) sred[g][tid >> 5] = s;
        }
        __syncthreads();
        if (tid < G) {
            float s = 0.f;
            for (int k = 0; k < kDecThreads / 32; ++k) s += sred[tid][k];
            ssum[tid] = ssum[tid] * salpha[tid] + s;
        }
        if constexpr (NSN) {
            // sum of e ||x|| / sqrt(d) over each block of the tile: token tid is in block tid / 128
            __syncthreads();  // sred is reused
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float b = (mine && tb + tid < t1) ? sw[g][tid] * svg[tid] : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
                if ((tid & 31) == 0) sred[g][tid >> 5] = b;
            }
            __syncthreads();
            if (tid < G * NBT) {
                const int g = tid / NBT, bq = tid % NBT;
                float b = 0.f;
                for (int k = bq * 4; k < bq * 4 + 4 && k < kDecThreads / 32; ++k) b += sred[g][k];
                sbeta[g][bq] = b;
            }
            __syncthreads();
        }
        // ---- phase C: value sums, one coordinate (or QJL row) per thread ----
        const int ntok = static_cast<int>(min(static_cast<int64_t>(TT), t1 - tb > 0 ? t1 - tb : 0));
#pragma unroll
        for (int g = 0; g < G; ++g) {
            accA[g] *= salpha[g];
            accB[g] *= salpha[g];
            accA2[g] *= salpha[g];
            accB2[g] *= salpha[g];
        }
        for (int role = tid; role < D + (QJL ? M : 0); role += kDecThreads) {
            const bool second = role >= kDecThreads;
            if (role < D) {
                const int j = role;
                float acc[G];
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = 0.f;
                for (int tt = 0; tt < ntok; ++tt) {
                    int code = 0;
#pragma unroll
                    for (int p = 0; p < B; ++p) code |= static_cast<int>((svc[tt >> 5][p][j] >> (tt & 31)) & 1u) << p;
                    const float c = scb[code] * svn[tt];
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[g] = fmaf(sw[g][tt], c, acc[g]);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    if (second) accA2[g] += acc[g];
                    else accA[g] += acc[g];
                }
                if constexpr (NSN) {
                    // O_j += sum over the tile's blocks of beta o_v,blk[j] (second vector of the partial)
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float o = 0.f;
                        for (int bq = 0; bq < NBT; ++bq) {
                            const int64_t blk = tb / 128 + bq;
                            if (blk * 128 < t1) o = fmaf(sbeta[g][bq], vmean_at(blk, j), o);
                        }
                        if (second) accB2[g] += o;
                        else accB[g] += o;
                    }
                }
            } else {
                const int i = role - D;
                float acc[G];
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = 0.f;
                for (int tt = 0; tt < ntok; ++tt) {
                    const float s = ((svq[tt >> 5][i] >> (tt & 31)) & 1u) ? 1.f : -1.f;
                    const float c = s * svn[tt] * svg[tt];
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[g] = fmaf(sw[g][tt], c, acc[g]);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    if (second) accB2[g] += acc[g];
                    else accB[g] += acc[g];
                }
            }
        }
        __syncthreads();
    }

    // ---- partials: {M, L, A[D], B[M]} per query head ----
    for (int role = tid, k = 0; role < D + (QJL ? M : 0); role += kDecThreads, ++k) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float* pp = a.part + ((qh0 + g) * a.nsplit + split) * PART;
            if (role < D) {
                pp[2 + role] = k ? accA2[g] : accA[g];
                if (NSN) pp[2 + D + role] = k ? accB2[g] : accB[g];  // the block-mean term O
            } else {
                pp[2 + role] = k ? accB2[g] : accB[g];
            }
        }
    }
    if (tid < G) {
        float* pp = a.part + ((qh0 + tid) * a.nsplit + split) * PART;
        pp[0] = smax[tid];
        pp[1] = ssum[tid];
    }
}

__device__ __forceinline__ float load_any(const void* p, int dt, int64_t i) {
    if (dt == 0) return reinterpret_cast<const float*>(p)[i];
    const uint16_t u = reinterpret_cast<const uint16_t*>(p)[i];
    return dt == 1 ? __half2float(__ushort_as_half(u)) : __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// The full-precision residual window of one (sequence, query head) as one more
// split partial (NSNQuant section 4: the newest tokens stay unquantized until
// a block is flushed): exact fp32 logits of its fp16 keys, its own max M and
// sum L, and y = sum_t e_t v_t.  Stored so that the combine's arithmetic
// gives y back: A = H (delta .* y) (delta .* H A / d = y), or for NSN caches
// the block-mean slot O = y.  An empty window leaves M = -inf, L = 0.
template <int D, bool NSN>
__global__ void __launch_bounds__(kDecThreads) decode_window_kernel(const __grid_constant__ DecodeArgs a) {
    // G = hq / hkv query heads (CTAs) read the same KV head's window
    constexpr int PART = 2 + 2 * D;
    __shared__ float sq[D];
    __shared__ float sl[kMaxWindow];
    __shared__ float sy[D];
    __shared__ float sred[kDecThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t qh = blockIdx.x;  // bi * hq + head
    const int bi = static_cast<int>(qh / a.hq);
    const int hk = static_cast<int>((qh % a.hq) / a.G);
    const int64_t stream = static_cast<int64_t>(bi) * a.hkv + hk;
    const int n = static_cast<int>(min(max(static_cast<int64_t>(a.win_len[bi]), int64_t(0)), a.win_cap));
    const __half* kw = a.kwin + stream * a.win_cap * D;
    const __half* vw = a.vwin + stream * a.win_cap * D;
    for (int j = tid; j < D; j += blockDim.x) sq[j] = load_any(a.q, a.qdtype, qh * D + j);
    __syncthreads();
    // logits, one token per thread (the key row in 16-byte loads)
    float mx = -INFINITY;
    for (int t = tid; t < n; t += blockDim.x) {
        const uint4* kr = reinterpret_cast<const uint4*>(kw + static_cast<int64_t>(t) * D);
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
            const uint4 w = kr[c];
            const __half2* hw = reinterpret_cast<const __half2*>(&w);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 kv = __half22float2(hw[k]);
                acc = fmaf(kv.y, sq[8 * c + 2 * k + 1], fmaf(kv.x, sq[8 * c + 2 * k], acc));
            }
        }
        const float l = a.scale * acc;
        sl[t] = l;
        mx = fmaxf(mx, l);
        if (a.logits != nullptr) a.logits[qh * a.logits_ld + a.max_T + t] = l;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0) sred[warp] = mx;
    __syncthreads();
    mx = sred[0];
    for (int w = 1; w < kDecThreads / 32; ++w) mx = fmaxf(mx, sred[w]);
    float sum = 0.f;
    for (int t = tid; t < n; t += blockDim.x) {
        const float e = __expf(sl[t] - mx);
        sl[t] = e;
        sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    __syncthreads();  // every thread has read sred (the max)
    if (lane == 0) sred[warp] = sum;
    __syncthreads();
    float L = 0.f;
    for (int w = 0; w < kDecThreads / 32; ++w) L += sred[w];
    // y = sum_t e_t v_t, one coordinate per thread (coalesced rows of V)
    for (int j = tid; j < D; j += blockDim.x) {
        float acc = 0.f;
        for (int t = 0; t < n; ++t) acc = fmaf(sl[t], __half2float(vw[static_cast<int64_t>(t) * D + j]), acc);
        sy[j] = NSN ? acc : sign_of(a.pair_sign, j) * acc;
    }
    __syncthreads();
    if (!NSN) fwht_smem<D>(sy);  // A = H (delta .* y)
    float* pp = a.part + (qh * a.nsplit + (a.nsplit - 1)) * PART;
    for (int j = tid; j < D; j += blockDim.x) {
        pp[2 + j] = NSN ? 0.f : sy[j];
        pp[2 + D + j] = NSN ? sy[j] : 0.f;
    }
    if (tid == 0) {
        pp[0] = n > 0 ? mx : -INFINITY;
        pp[1] = n > 0 ? L : 0.f;
    }
}

// Merge the splits of one (batch, query head) and rotate back.  NSN: the
// second vector of each partial is the block-mean term O (no QJL), added
// after the inverse rotation: out = delta .* H A / (d L) + O / L.
template <int D, bool QJL, bool NSN = false>
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int M = D;
    constexpr int PART = 2 + D + M;
    __shared__ float sA[D], sB[M];
    __shared__ float sf[512];
    __shared__ float sred[kDecThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t bh = blockIdx.x;
    const int ns = a.nsplit;
    const float* pp = a.part + bh * ns * PART;
    // block-wide max (op 0) or sum (op 1) of one value per thread
    auto block_reduce = [&](float v, int op) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
            v = op == 0 ? fmaxf(v, w) : v + w;
        }
        __syncthreads();  // sred is free (an earlier reduction has been read)
        if (lane == 0) sred[wid] = v;
        __syncthreads();
        float r = sred[0];
        for (int k = 1; k < kDecThreads / 32; ++k) r = op == 0 ? fmaxf(r, sred[k]) : r + sred[k];
        return r;
    };
    // running max over the splits that saw tokens, then L = sum_s e^(M_s - max) L_s
    float mx = -INFINITY;
    for (int s = tid; s < ns; s += blockDim.x)
        if (pp[s * PART + 1] > 0.f) mx = fmaxf(mx, pp[s * PART]);
    mx = block_reduce(mx, 0);
    float lp = 0.f;
    for (int s = tid; s < ns; s += blockDim.x)
        if (pp[s * PART + 1] > 0.f) lp += __expf(pp[s * PART] - mx) * pp[s * PART + 1];
    const float L = block_reduce(lp, 1);
    if (!(L > 0.f)) {
        for (int j = tid; j < D; j += blockDim.x) a.out[bh * D + j] = 0.f;
        return;
    }
    // weighted sums of A and B over the splits, 512 split factors at a time
    constexpr int EXTRA = (QJL || NSN) ? M : 0;  // entries of the second vector
    constexpr int NE = (D + EXTRA + kDecThreads - 1) / kDecThreads;
    float acc[NE];
#pragma unroll
    for (int k = 0; k < NE; ++k) acc[k] = 0.f;
    for (int c0 = 0; c0 < ns; c0 += 512) {
        const int nc = min(512, ns - c0);
        for (int s = tid; s < nc; s += blockDim.x) {
            const float* ps = pp + static_cast<int64_t>(c0 + s) * PART;
            sf[s] = ps[1] > 0.f ? __expf(ps[0] - mx) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < NE; ++k) {
            const int e = tid + k * kDecThreads;
            if (e < D + EXTRA)
                for (int s = 0; s < nc; ++s) acc[k] = fmaf(sf[s], pp[static_cast<int64_t>(c0 + s) * PART + 2 + e], acc[k]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < NE; ++k) {
        const int e = tid + k * kDecThreads;
        if (e < D) sA[e] = acc[k];
        else if (e < D + EXTRA) sB[e - D] = acc[k];
    }
    __syncthreads();
    // v = A + sqrt(pi/2)/m S^T B, in place in sA
    float vj[(D + kDecThreads - 1) / kDecThreads];
    int k = 0;
    for (int j = threadIdx.x; j < D; j += blockDim.x, ++k) {
        float v = sA[j];
        if (QJL) {
            float st = 0.f;
            for (int i = 0; i < M; ++i) st = fmaf(__half2float(a.S[static_cast<int64_t>(i) * D + j]), sB[i], st);
            v = fmaf(kSqrtHalfPi / M, st, v);
        }
        vj[k] = v;
    }
    __syncthreads();
    k = 0;
    for (int j = threadIdx.x; j < D; j += blockDim.x, ++k) sA[j] = vj[k];
    __syncthreads();
    fwht_smem<D>(sA);
    const float inv = 1.0f / (static_cast<float>(D) * L);
    for (int j = threadIdx.x; j < D; j += blockDim.x)
        a.out[bh * D + j] = sign_of(a.pair_sign, j) * sA[j] * inv + (NSN ? sB[j] / L : 0.f);
}

template <int D, int B, bool QJL>
cudaError_t launch_d(const DecodeArgs& a, cudaStream_t s) {
    const dim3 block(kDecThreads);
    const int nbh = a.batch * a.hq;
    switch (a.qdtype) {
        case 0: qproj_kernel<D, 0, QJL><<<nbh, block, 0, s>>>(a); break;
        case 1: qproj_kernel<D, 1, QJL><<<nbh, block, 0, s>>>(a); break;
        default: qproj_kernel<D, 2, QJL><<<nbh, block, 0, s>>>(a); break;
    }
    const dim3 grid(a.nsplit_run, a.hkv, a.batch);
    bool nsn = false;
    if constexpr (!QJL) nsn = a.nsn != 0;
    if (nsn) {
        if constexpr (!QJL) {
            auto run = [&](auto dq) {
                constexpr bool DQ = decltype(dq)::value;
                switch (a.G) {
                    case 1: decode_split_kernel<D, B, false, 1, true, DQ><<<grid, block, 0, s>>>(a); break;
                    case 2: decode_split_kernel<D, B, false, 2, true, DQ><<<grid, block, 0, s>>>(a); break;
                    case 4: decode_split_kernel<D, B, false, 4, true, DQ><<<grid, block, 0, s>>>(a); break;
                    default: decode_split_kernel<D, B, false, 8, true, DQ><<<grid, block, 0, s>>>(a); break;
                }
            };
            if (a.nsn_dq) run(std::true_type());
            else run(std::false_type());
        }
    } else {
        switch (a.G) {
            case 1: decode_split_kernel<D, B, QJL, 1><<<grid, block, 0, s>>>(a); break;
            case 2: decode_split_kernel<D, B, QJL, 2><<<grid, block, 0, s>>>(a); break;
            case 4: decode_split_kernel<D, B, QJL, 4><<<grid, block, 0, s>>>(a); break;
            default: decode_split_kernel<D, B, QJL, 8><<<grid, block, 0, s>>>(a); break;
        }
    }
    if (a.kwin != nullptr) {
        const cudaError_t e = launch_decode_window(nullptr, a, s);
        if (e != cudaSuccess) return e;
    }
    if (nsn) decode_combine_kernel<D, false, true><<<nbh, block, 0, s>>>(a);
    else decode_combine_kernel<D, QJL><<<nbh, block, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, int B>
cudaError_t launch_db(const DecodeArgs& a, bool qjl, cudaStream_t s) {
    return qjl ? launch_d<D, B, true>(a, s) : launch_d<D, B, false>(a, s);
}

template <int D>
cudaError_t launch_dd(const DecodeArgs& a, int b, bool qjl, cudaStream_t s) {
    switch (b) {
        case 1: return launch_db<D, 1>(a, qjl, s);
        case 2: return launch_db<D, 2>(a, qjl, s);
        case 3: return launch_db<D, 3>(a, qjl, s);
        default: return launch_db<D, 4>(a, qjl, s);
    }
}

}  // namespace

void decode_plan(const kvq_ctx* h, int batch, int hq, int hkv, int64_t max_T, int* nsplit, int64_t* chunk,
                 size_t* ws_bytes) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
    const int64_t streams = static_cast<int64_t>(batch) * hkv;
    int64_t ch;
    if (decode_uses_mma(h)) {
        // Persistent grid over (stream, split) items: about 16 items per
        // resident CTA keeps the last round short; splits are multiples of 256
        // tokens and at least 1024 (amortising the per-item set-up).  When even
        // 1024-token splits leave fewer than 3 rounds of items over the grid
        // (few streams), a short last round costs a large share of the call:
        // then the split is the one, up to 4x longer, whose rounds cost least,
        // counting an item as its tokens plus a set-up worth kItemCost tokens.
        constexpr int64_t kItemCost = 384;
        const int64_t grid = decode_mma_grid(h, hkv > 0 ? hq / hkv : 1);
        const int64_t g = grid > 0 ? grid : 1;
        const int64_t target = 16 * g;
        int64_t lo = (streams * max_T + target - 1) / target;
        lo = (lo + 255) / 256 * 256;
        if (lo < 1024) lo = 1024;
        ch = lo;
        if (streams * ((max_T + lo - 1) / lo) < 3 * g) {
            const int64_t mx = (max_T + 255) / 256 * 256;
            int64_t best_cost = -1;
            for (int64_t c = lo; c <= 4 * lo && (c == lo || c <= mx); c += 256) {
                const int64_t rounds = (streams * ((max_T + c - 1) / c) + g - 1) / g;
                const int64_t cost = rounds * (c + kItemCost);
                if (best_cost < 0 || cost < best_cost) {
                    ch = c;
                    best_cost = cost;
                }
            }
        }
        if ((max_T + ch - 1) / ch > 4096) ch = ((max_T + 4095) / 4096 + 255) / 256 * 256;
    } else {
        int64_t want = (4 * static_cast<int64_t>(sms) + streams - 1) / (streams > 0 ? streams : 1);
        const int64_t tiles = (max_T + kTokTile - 1) / kTokTile;
        if (want > tiles) want = tiles;
        if (want > 512) want = 512;
        if (want < 1) want = 1;
        ch = (max_T + want - 1) / want;
        ch = (ch + kTokTile - 1) / kTokTile * kTokTile;
        if (ch < kTokTile) ch = kTokTile;
    }
    const int64_t ns = (max_T + ch - 1) / ch > 0 ? (max_T + ch - 1) / ch : 1;
    *nsplit = static_cast<int>(ns);
    *chunk = ch;
    const int64_t bh = static_cast<int64_t>(batch) * hq;
    // partials first (both paths; one more split for a residual window), then
    // the path's query data
    size_t bytes = static_cast<size_t>(bh * (ns + 1) * (2 + h->d + h->m)) * sizeof(float);
    bytes = (bytes + 255) / 256 * 256;
    if (decode_uses_mma(h)) {
        bytes += static_cast<size_t>(bh) * 4 * sizeof(float);
        bytes = (bytes + 255) / 256 * 256;
        bytes += static_cast<size_t>(streams) * decode_mma_qfrag_bytes(h, hq / hkv);
    } else {
        bytes += static_cast<size_t>(bh) * (h->d + h->m) * sizeof(float);
    }
    *ws_bytes = bytes + 256;
}

cudaError_t launch_decode(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s, std::string* why) {
    const bool qjl = (h->flags & 1u) != 0;
    if (decode_uses_mma(h)) {
        cudaError_t e = launch_decode_mma(h, a, s);
        if (e != cudaSuccess) return e;
        if (a.kwin != nullptr) {
            e = launch_decode_window(h, a, s);
            if (e != cudaSuccess) return e;
        }
        const unsigned nbh = static_cast<unsigned>(a.batch * a.hq);
        switch (h->d) {
            case 64:
                if (a.nsn) decode_combine_kernel<64, false, true><<<nbh, kDecThreads, 0, s>>>(a);
                else if (qjl) decode_combine_kernel<64, true><<<nbh, kDecThreads, 0, s>>>(a);
                else decode_combine_kernel<64, false><<<nbh, kDecThreads, 0, s>>>(a);
                break;
            case 128:
                if (a.nsn) decode_combine_kernel<128, false, true><<<nbh, kDecThreads, 0, s>>>(a);
                else if (qjl) decode_combine_kernel<128, true><<<nbh, kDecThreads, 0, s>>>(a);
                else decode_combine_kernel<128, false><<<nbh, kDecThreads, 0, s>>>(a);
                break;
            default:
                if (a.nsn) decode_combine_kernel<256, false, true><<<nbh, kDecThreads, 0, s>>>(a);
                else if (qjl) decode_combine_kernel<256, true><<<nbh, kDecThreads, 0, s>>>(a);
                else decode_combine_kernel<256, false><<<nbh, kDecThreads, 0, s>>>(a);
                break;
        }
        return cudaGetLastError();
    }
    switch (h->d) {
        case 64: return launch_dd<64>(a, h->b, qjl, s);
        case 128: return launch_dd<128>(a, h->b, qjl, s);
        case 256: return launch_dd<256>(a, h->b, qjl, s);
        default:
            if (why) *why = "unsupported head dimension";
            return cudaErrorInvalidValue;
    }
}

namespace {
template <int D>
cudaError_t window_d(const DecodeArgs& a, cudaStream_t s) {
    const unsigned n = static_cast<unsigned>(a.batch * a.hq);
    if (a.nsn) decode_window_kernel<D, true><<<n, kDecThreads, 0, s>>>(a);
    else decode_window_kernel<D, false><<<n, kDecThreads, 0, s>>>(a);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_decode_window(const kvq_ctx*, const DecodeArgs& a, cudaStream_t s) {
    const int D = static_cast<int>(a.win_dim);
    switch (D) {
        case 64: return window_d<64>(a, s);
        case 128: return window_d<128>(a, s);
        default: return window_d<256>(a, s);
    }
}

// The bounded-wait path on its own: one thread waits on an mbarrier that no
// one arrives on, for `polls` polls, then records the timeout in the status
// word and returns (the same helper every kernel's waits use).
__global__ void wait_timeout_probe_kernel(uint32_t* status, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait_n(&bar, 0u, status, polls);
    }
}

cudaError_t launch_wait_timeout_probe(uint32_t* status, uint32_t polls, cudaStream_t s) {
    wait_timeout_probe_kernel<<<1, 32, 0, s>>>(status, polls);
    return cudaGetLastError();
}

}  // namespace kvq
