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
__device__ __forceinline__ float prepare_dt(float raw, int h, const DtPreArgs &p) {
    float v = raw + (p.bias ? p.bias[h] : 0.f);
    if (p.softplus) v = fmaxf(v, 0.f) + log1pf(expf(-fabsf(v)));
    if (p.dt_max > 0.f) v = fminf(fmaxf(v, p.dt_min), p.dt_max);
    return v;
}

// Input weight of a prepared step: dt, or (exp(dt A) - 1) / A under the
// zero-order hold (dt where A = 0).
__device__ __forceinline__ float input_weight(float dt, float A, int zoh) {
    return (zoh && A != 0.f) ? expm1f(dt * A) / A : dt;
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
