// kla_device.cuh -- small device helpers shared by the KLA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kla {

constexpr int kChunk = 64;  // chunk length C of the chunkwise form

// Element load/store for the two supported input types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// The Kaczmarz coefficient written on unit keys (section 3.1, Eq. (3), with k = r * khat):
//   beta k e^T = (eta r^2/(r^2+eps)) khat (v/r - Sbar^T khat)^T
// so the write uses khat with coefficient b = eta r^2/(r^2+eps) on the state term and
// c = eta r/(r^2+eps) on the value term.  Both are zero when r^2 + eps == 0 (write skipped).
struct KaczCoef {
    float b, c, inv_r;
};
// eps < 0 is never a Kaczmarz stabiliser (the C ABI rejects it): the library passes
// kBetaDirect to the kernels to select the direct write strength beta = eta as given.
constexpr float kBetaDirect = -1.f;
// Coefficients of the unit-key form (k = r khat): the write beta k k^T = b khat khat^T and the
// value injection beta k = c khat.  Kaczmarz (Eq. 3): beta = eta / (r^2 + eps), so
// b = eta r^2 / (r^2 + eps), c = eta r / (r^2 + eps); direct: beta = eta, b = eta r^2, c = eta r.
// A zero key writes nothing in either mode.
__device__ __forceinline__ KaczCoef kacz_coef(float eta, float r2, float eps) {
    KaczCoef out;
    const float r = sqrtf(r2);
    if (eps < 0.f) {
        if (r > 0.f) {
            out.b = eta * r2;
            out.c = eta * r;
            out.inv_r = 1.f / r;
        } else {
            out.b = out.c = out.inv_r = 0.f;
        }
        return out;
    }
    float den = r2 + eps;
    if (den > 0.f && r > 0.f) {
        out.b = eta * r2 / den;
        out.c = eta * r / den;
        out.inv_r = 1.f / r;
    } else {
        out.b = 0.f;
        out.c = 0.f;
        out.inv_r = 0.f;
    }
    return out;
}

}  // namespace kla
