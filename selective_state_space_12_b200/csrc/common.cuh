// Device helpers shared by the libssd kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
// Round to nearest, ties to even.
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Four consecutive elements as floats (16-byte load for fp32, 8-byte for bf16).
template <typename T> __device__ __forceinline__ float4 load4(const T *p);
template <> __device__ __forceinline__ float4 load4<float>(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    float4 r;
    r.x = __uint_as_float(u.x << 16);
    r.y = __uint_as_float(u.x & 0xffff0000u);
    r.z = __uint_as_float(u.y << 16);
    r.w = __uint_as_float(u.y & 0xffff0000u);
    return r;
}

// Step options in kernel arguments (the host's DtPre): raw -> + bias ->
// softplus -> clamp (dt_max > 0); input weight dt or the zero-order hold.
struct DtPreArgs {
    const float *bias;
    int softplus, zoh;
    float dt_min, dt_max;
};

// The prepared step of one raw value of head h. softplus(v) is written as
// max(v, 0) + log1p(exp(-|v|)) so that exp cannot overflow.
__device__ __forceinline__ float prepare_dt(float raw, float bias_h, const DtPreArgs &p) {
    float v = raw + bias_h;
    if (p.softplus) v = fmaxf(v, 0.f) + log1pf(expf(-fabsf(v)));
    if (p.dt_max > 0.f) v = fminf(fmaxf(v, p.dt_min), p.dt_max);
    return v;
}
__device__ __forceinline__ float prepare_dt(float raw, int h, const DtPreArgs &p) {
    return prepare_dt(raw, p.bias ? p.bias[h] : 0.f, p);
}

// Input weight of a prepared step: dt, or (exp(dt A) - 1) / A under the
// zero-order hold (dt where A = 0).
__device__ __forceinline__ float input_weight(float dt, float A, int zoh) {
    return (zoh && A != 0.f) ? expm1f(dt * A) / A : dt;
}

// Compact forms of the step preparation for the bf16 tensor-core kernel,
// whose hot code must stay small (the accurate library functions carry long
// rarely-taken paths). Both are Taylor expansions plus the hardware exp2 /
// log2 units, with relative error below ~3e-5 (bf16 I/O keeps ~4e-3):
//
//   log1p(e), e in (0, 1]:  e < 2^-6: e - e^2/2 + e^3/3 - e^4/4 (the next
//                           term is below e^5/5 < 2^-30 e); otherwise
//                           log(1 + e) by the hardware log (absolute error
//                           about 2^-21 on [1, 2], against log1p(e) >= 2^-6)
//   expm1(x):               |x| < 1/2: x (1 + x/2 + x^2/6 + ... + x^6/5040)
//                           (remainder below x^7/40320 < 2e-7 relative);
//                           otherwise exp(x) - 1, where |exp(x) - 1| > 0.39
__device__ __forceinline__ float softplus_compact(float v) {
    const float e = __expf(-fabsf(v));
    const float series = e * fmaf(e, fmaf(e, fmaf(e, -0.25f, 1.f / 3.f), -0.5f), 1.f);
    const float l = (e < 0.015625f) ? series : __logf(1.f + e);
    return fmaxf(v, 0.f) + l;
}

__device__ __forceinline__ float expm1_compact(float x) {
    float q = 1.f / 5040.f;
    q = fmaf(q, x, 1.f / 720.f);
    q = fmaf(q, x, 1.f / 120.f);
    q = fmaf(q, x, 1.f / 24.f);
    q = fmaf(q, x, 1.f / 6.f);
    q = fmaf(q, x, 0.5f);
    q = fmaf(q, x, 1.f);
    return (fabsf(x) < 0.5f) ? x * q : __expf(x) - 1.f;
}

// prepare_dt / input_weight with the compact forms; inv_A = 1 / A (0 when A = 0).
__device__ __forceinline__ float prepare_dt_compact(float raw, float bias_h, const DtPreArgs &p) {
    float v = raw + bias_h;
    if (p.softplus) v = softplus_compact(v);
    if (p.dt_max > 0.f) v = fminf(fmaxf(v, p.dt_min), p.dt_max);
    return v;
}
__device__ __forceinline__ float input_weight_compact(float dt, float A, float inv_A, int zoh) {
    return (zoh && A != 0.f) ? expm1_compact(dt * A) * inv_A : dt;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive prefix sum over a block of up to 1024 threads; `warp_tot` is
// shared scratch of 32 floats. Every thread of the block must call it.
__device__ __forceinline__ float block_inclusive_scan(float v, float *warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float t = lane < nwarps ? warp_tot[lane] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        if (lane < nwarps) warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    __syncthreads();
    return v;
}

}  // namespace ssd
