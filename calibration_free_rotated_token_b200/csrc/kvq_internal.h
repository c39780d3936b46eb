// kvq_internal.h -- handle layout and kernel-launch interfaces shared by the
// C-ABI layer (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <vector>

struct kvq_ctx {
    int device = 0;
    int d = 0, b = 0, m = 0;
    uint32_t flags = 0;
    uint64_t seed = 0;
    // Host copies of the constants.
    std::vector<int8_t> signs;        // [d]
    std::vector<uint16_t> S_half;     // [m][d] fp16 patterns
    std::vector<float> centroids;     // [2^b]
    std::vector<float> thresholds;    // [2^b - 1]
    // Sign masks of bf16/fp16 pairs: bit 15 = sign of coordinate 2k, bit 31 =
    // sign of coordinate 2k+1 (1 = negative).  XOR flips both halves' signs.
    uint32_t pair_sign[128] = {};
    // Device constants.
    __half* d_S = nullptr;            // [m][d]
    uint32_t* d_status = nullptr;     // one word, ORed by kernels
    // Resident CTAs of the tensor-core decode kernel per group size G (index
    // G = 1, 2, 4, 8; 0 = not yet queried).
    int mma_grid[9] = {};
};

namespace kvq {

constexpr int kTileRows = 128;        // vectors per MMA tile (M of the S.r product)
constexpr int kMaxLevels = 16;

// Everything a quantize kernel needs besides the TMA tensor map.  Passed by
// value as a __grid_constant__ parameter (lives in the constant bank).
struct QuantArgs {
    int64_t n;                        // vectors (rows)
    int layout;                       // 0: one record per vector, 1: blocks of 32 vectors transposed
    int64_t ntiles;
    uint32_t* codes;                  // [n][b][d/32]
    uint32_t* qjl;                    // [n][d/32] or null
    __half2* norms;                   // [n]
    __half* block_mean;               // NSN: [n/128][d]
    uint8_t* side;                    // NSN with double quantization: one side record per 128 rows (else null)
    int cuda_core_rotation;           // plain 16-bit input: the in-register transform kernel instead of tcgen05
    const __half* S;                  // [m][d] fp16 (global), copied to smem per CTA
    uint32_t* status;
    float centroid[kMaxLevels];
    float threshold[kMaxLevels];
    uint32_t pair_sign[128];
    // A second stream of vectors in the same launch (tensor-core kernel
    // only): tiles [ntiles0, ntiles) read the second tensor map and write
    // these outputs.  With one stream ntiles0 = ntiles.
    int64_t ntiles0;
    int64_t n1;
    int layout1;
    uint32_t* codes1;
    uint32_t* qjl1;
    __half2* norms1;
};

// Launch the quantizer (nsn = false) or the NSN front end + quantizer
// (nsn = true) over n rows described by `map` (2-D TMA map, 128-byte swizzle,
// box = 128 bytes x 128 rows).  Returns a cudaError_t.
cudaError_t launch_quantize(const kvq_ctx* h, const CUtensorMap& map, int dtype, bool nsn, const QuantArgs& a,
                            cudaStream_t s, std::string* why);
// True when two streams of vectors can share one launch (the tensor-core
// kernel: 16-bit input, no NSN front end, d <= 128 or d = 256 without QJL).
inline bool quantize_pairs(int d, int dtype, bool nsn, bool qjl) { return dtype != 0 && !nsn && (d <= 128 || !qjl); }

struct DecodeArgs {
    int batch, hq, hkv, G;            // G = hq / hkv
    int64_t max_T;
    int nsplit;
    int64_t chunk;                    // tokens per split
    const void* q;
    int qdtype;
    const uint32_t* kcodes;
    const uint32_t* kqjl;
    const __half2* knorms;
    const uint32_t* vcodes;
    const uint32_t* vqjl;
    const __half2* vnorms;
    int64_t kcap, vcap;               // vectors per stream
    const int32_t* seq_len;
    float scale;
    float* logits;                    // nullable
    float* out;
    float* qrot;                      // workspace [batch*hq][d]   q' = H (delta.*q)
    float* qproj;                     // workspace [batch*hq][m]   p = S q'
    float* part;                      // workspace [batch*hq][nsplit][2 + d + m]
    uint2* qfrag;                     // tensor path: workspace, query fragments per (sequence, KV head)
    uint32_t* status;                 // device status word of the handle
    float* qscal;                     // tensor path: workspace [batch*hq][4] per-head scalars
    const __half* S;
    float centroid[kMaxLevels];
    uint32_t pair_sign[128];
    // NSN caches (no QJL): fp16 block means, [capacity / 128][d] per stream;
    // the partials' second vector then holds the block-mean term O.
    int nsn;
    const __half* kmean;
    const __half* vmean;
    // NSN caches with double-quantized side data: the norms arrays hold fp16
    // ||w|| per token and kmean / vmean point at the side records.
    int nsn_dq;
    // Splits over the packed cache (nsplit counts one more when a window is
    // attended: its partial is split nsplit - 1); row stride of `logits`.
    int nsplit_run;
    int64_t logits_ld;
    // Full-precision residual window (optional): fp16 [streams][win_cap][d]
    // keys and values, win_len[batch] tokens each.
    const __half* kwin;
    const __half* vwin;
    int64_t win_cap;
    const int32_t* win_len;
    int win_dim;                      // d of the handle (selects the window kernel)
};

constexpr int kMaxWindow = 256;  // tokens of a residual window (KVQ_MAX_WINDOW)

// One bounded mbarrier wait that cannot complete (a test of the timeout path).
cudaError_t launch_wait_timeout_probe(uint32_t* status, uint32_t polls, cudaStream_t s);

// Exact attention partial of the residual window for every (sequence, query head).
cudaError_t launch_decode_window(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s);

// Bytes of workspace and number of splits for a decode of these sizes.
void decode_plan(const kvq_ctx* h, int batch, int hq, int hkv, int64_t max_T, int* nsplit, int64_t* chunk,
                 size_t* ws_bytes);

cudaError_t launch_decode(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s, std::string* why);

// Tensor-core decode path (1- and 2-bit codebooks, and 3-bit at d <= 128): query fragments + split kernel.
cudaError_t launch_decode_mma(const kvq_ctx* h, const DecodeArgs& a, cudaStream_t s);
size_t decode_mma_qfrag_bytes(const kvq_ctx* h, int G);
// Resident CTAs of the tensor-core split kernel on the device (its persistent grid).
int decode_mma_grid(const kvq_ctx* h, int G);
// 3-bit codebooks take four code planes (the parity plane included); at
// d = 256 their operands no longer fit the register file, so they stay on the
// CUDA-core path there.
inline bool decode_uses_mma(const kvq_ctx* h) { return h->b <= 2 || (h->b == 3 && h->d <= 128); }

// Size of the fixed scratch of kvq_decode_attend_noalloc (mirrors
// KVQ_NOALLOC_SCRATCH_BYTES of kvq.h) and its address on `device`, which
// must be the current device.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
cudaError_t noalloc_scratch(int device, void** ptr);

}  // namespace kvq
