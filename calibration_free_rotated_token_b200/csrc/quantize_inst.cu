// quantize_inst.cu -- instantiates the quantize kernels of one (d, b), given
// as -DKVQ_D=<d> -DKVQ_B=<b> by the build; the build compiles this file once
// per supported pair so that the twelve instantiations compile in parallel.
// 16-bit input takes the tensor-core rotation kernel (quantize_tc.cuh), with
// or without the NSN front end, except at d = 256 with QJL; fp32 input and
// d = 256 with QJL take the kernel with the in-register transform
// (quantize.cuh), which plain 16-bit input takes too when the handle asks for
// the CUDA-core rotation.
#include "quantize_tc.cuh"

#ifndef KVQ_D
#error "KVQ_D must be defined"
#endif
#ifndef KVQ_B
#error "KVQ_B must be defined"
#endif

#define KVQ_CAT4(a, b, c, d) a##b##c##d
#define KVQ_LAUNCH_NAME(D, B) KVQ_CAT4(launch_quantize_d, D, _b, B)

namespace kvq {

namespace {

template <int D, int B, bool QJL, bool NSN>
cudaError_t by_dtype(const CUtensorMap& map, const CUtensorMap& map1, int dtype, const QuantArgs& a, int sms,
                     cudaStream_t s) {
    if constexpr (NSN && QJL) {
        return cudaErrorNotSupported;
    } else if constexpr (NSN) {
        // double-quantized side data (a.side): 16-bit input only
        if (a.side != nullptr) {
            switch (dtype) {
                case DT_F16: return launch_quantize_tc<D, B, false, DT_F16, true, true>(map, map1, a, sms, s);
                case DT_BF16: return launch_quantize_tc<D, B, false, DT_BF16, true, true>(map, map1, a, sms, s);
                default: return cudaErrorNotSupported;
            }
        }
        switch (dtype) {
            case DT_F32:
                if constexpr (D <= 128) return launch_quantize_t<D, B, false, DT_F32, true>(map, a, sms, s);
                else return cudaErrorNotSupported;
            case DT_F16: return launch_quantize_tc<D, B, false, DT_F16, true>(map, map1, a, sms, s);
            default: return launch_quantize_tc<D, B, false, DT_BF16, true>(map, map1, a, sms, s);
        }
    } else {
        // the tensor-core rotation is built for d <= 128, and for d = 256 without QJL
        constexpr bool kTc = D <= 128 || !QJL;
        switch (dtype) {
            case DT_F32:
                if constexpr (D <= 128) return launch_quantize_t<D, B, QJL, DT_F32, false>(map, a, sms, s);
                else return cudaErrorNotSupported;
            case DT_F16:
                if constexpr (kTc) {
                    if (a.cuda_core_rotation) return launch_quantize_t<D, B, QJL, DT_F16, false>(map, a, sms, s);
                    return launch_quantize_tc<D, B, QJL, DT_F16>(map, map1, a, sms, s);
                } else {
                    return launch_quantize_t<D, B, QJL, DT_F16, false>(map, a, sms, s);
                }
            default:
                if constexpr (kTc) {
                    if (a.cuda_core_rotation) return launch_quantize_t<D, B, QJL, DT_BF16, false>(map, a, sms, s);
                    return launch_quantize_tc<D, B, QJL, DT_BF16>(map, map1, a, sms, s);
                } else {
                    return launch_quantize_t<D, B, QJL, DT_BF16, false>(map, a, sms, s);
                }
        }
    }
}

}  // namespace

// map1 describes the second stream of vectors (tiles [a.ntiles0, a.ntiles));
// only the tensor-core kernel takes two streams (quantize_pairs).
cudaError_t KVQ_LAUNCH_NAME(KVQ_D, KVQ_B)(bool qjl, bool nsn, const CUtensorMap& map, const CUtensorMap& map1,
                                           int dtype, const QuantArgs& a, int sms, cudaStream_t s) {
    if (a.ntiles0 != a.ntiles && !quantize_pairs(KVQ_D, dtype, nsn, qjl)) return cudaErrorNotSupported;
    if (nsn) return by_dtype<KVQ_D, KVQ_B, false, true>(map, map1, dtype, a, sms, s);
    return qjl ? by_dtype<KVQ_D, KVQ_B, true, false>(map, map1, dtype, a, sms, s)
               : by_dtype<KVQ_D, KVQ_B, false, false>(map, map1, dtype, a, sms, s);
}

}  // namespace kvq
