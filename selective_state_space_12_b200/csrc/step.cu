// One-token decode step, in place ("Mamba-2 — 注意力的远亲", section
// "跟着四个 token 算一次": the recurrent form carries a fixed-size state and
// serves generation):
//
//   a = exp(dt A_h);  h[p][n] = a h[p][n] + w x[p] B[g][n];
//   y[p] = sum_n C[g][n] h[p][n] + D_h x[p]
//
// with w = dt, or the zero-order hold (exp(dt A_h) - 1) / A_h, and dt the raw
// step prepared by the step options (common.cuh: prepare_dt, input_weight).
//
// Bound by HBM: the fp32 state is read once and written once. One block per
// (b, h); one warp per state row (p), each lane one 16-byte vector of the row
// per 128 state entries; rows are processed four at a time so that four
// 16-byte loads per lane are in flight before any arithmetic.
#include "common.cuh"
#include "internal.h"

namespace ssd {
namespace {

constexpr int kStepThreads = 256;
constexpr int kRows = 4;  // rows in flight per warp (generic kernel)

// Generic kernel: any N that is a multiple of 4 up to 256.
template <typename T>
__global__ void __launch_bounds__(kStepThreads)
step_kernel(float *__restrict__ h, const T *__restrict__ x, const T *__restrict__ dt,
            const float *__restrict__ A, const T *__restrict__ B, const T *__restrict__ C,
            const float *__restrict__ D, T *__restrict__ y, int H, int P, int N, int G,
            const DtPreArgs pre) {
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H), hh = (int)(bh % H), g = hh / (H / G);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const float dtv = prepare_dt(to_f(dt[bh]), hh, pre);
    const float a = expf(dtv * A[hh]);
    const float wv = input_weight(dtv, A[hh], pre.zoh);
    const float Dh = D ? D[hh] : 0.f;
    const int N4 = N >> 2;  // 16-byte vectors per row: 4..64
    const bool has0 = lane < N4, has1 = lane + 32 < N4;
    const T *Bp = B + ((int64_t)b * G + g) * N;
    const T *Cp = C + ((int64_t)b * G + g) * N;
    float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), c0 = b0, b1 = b0, c1 = b0;
    if (has0) {
        b0 = load4(Bp + 4 * lane);
        c0 = load4(Cp + 4 * lane);
    }
    if (has1) {
        b1 = load4(Bp + 4 * (lane + 32));
        c1 = load4(Cp + 4 * (lane + 32));
    }
    float *hb = h + bh * (int64_t)P * N;
    const T *xb = x + bh * P;
    T *yb = y + bh * P;
    for (int p0 = warp * kRows; p0 < P; p0 += nwarps * kRows) {
        float4 v0[kRows], v1[kRows];
        float xv[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const float4 *row = reinterpret_cast<const float4 *>(hb + (int64_t)(p0 + r) * N);
            if (has0) v0[r] = row[lane];
            if (has1) v1[r] = row[lane + 32];
            xv[r] = to_f(xb[p0 + r]);
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float4 *row = reinterpret_cast<float4 *>(hb + (int64_t)(p0 + r) * N);
            const float wx = wv * xv[r];
            float acc = 0.f;
            if (has0) {
                float4 v = v0[r];
                v.x = fmaf(a, v.x, wx * b0.x);
                v.y = fmaf(a, v.y, wx * b0.y);
                v.z = fmaf(a, v.z, wx * b0.z);
                v.w = fmaf(a, v.w, wx * b0.w);
                row[lane] = v;
                acc = v.x * c0.x + v.y * c0.y + v.z * c0.z + v.w * c0.w;
            }
            if (has1) {
                float4 v = v1[r];
                v.x = fmaf(a, v.x, wx * b1.x);
                v.y = fmaf(a, v.y, wx * b1.y);
                v.z = fmaf(a, v.z, wx * b1.z);
                v.w = fmaf(a, v.w, wx * b1.w);
                row[lane + 32] = v;
                acc += v.x * c1.x + v.y * c1.y + v.z * c1.z + v.w * c1.w;
            }
            acc = warp_sum(acc);
            if (lane == 0) yb[p0 + r] = from_f<T>(acc + Dh * xv[r]);
        }
    }
}

// N = 128 and head dim 64 (the common Mamba-2 shape): a row is exactly one
// 16-byte vector per lane, and each warp takes its eight rows in one pass,
// eight loads per lane in flight before any arithmetic. Compile-time shape,
// no idle lanes, no second vector set (62 registers: four blocks per SM).
template <typename T>
__global__ void __launch_bounds__(kStepThreads)
step_kernel_n128(float *__restrict__ h, const T *__restrict__ x, const T *__restrict__ dt,
                 const float *__restrict__ A, const T *__restrict__ B, const T *__restrict__ C,
                 const float *__restrict__ D, T *__restrict__ y, int H, int G,
                 const DtPreArgs pre) {
    constexpr int N = 128, P = 64, kWarps = kStepThreads / 32;
    static_assert(P % kWarps == 0, "rows per warp");
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H), hh = (int)(bh % H), g = hh / (H / G);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *hb = h + bh * (int64_t)P * N;
    // state loads first: they do not depend on anything else
    float4 v[P / kWarps];
#pragma unroll
    for (int r = 0; r < P / kWarps; ++r)
        v[r] = reinterpret_cast<const float4 *>(hb + (int64_t)(warp + kWarps * r) * N)[lane];
    const float dtv = prepare_dt(to_f(dt[bh]), hh, pre);
    const float a = expf(dtv * A[hh]);
    const float wv = input_weight(dtv, A[hh], pre.zoh);
    const float Dh = D ? D[hh] : 0.f;
    const float4 bv = load4(B + ((int64_t)b * G + g) * N + 4 * lane);
    const float4 cv = load4(C + ((int64_t)b * G + g) * N + 4 * lane);
    const T *xb = x + bh * P;
    T *yb = y + bh * P;
#pragma unroll
    for (int r = 0; r < P / kWarps; ++r) {
        const int p = warp + kWarps * r;
        const float xr = to_f(xb[p]);
        const float wx = wv * xr;
        float4 s = v[r];
        s.x = fmaf(a, s.x, wx * bv.x);
        s.y = fmaf(a, s.y, wx * bv.y);
        s.z = fmaf(a, s.z, wx * bv.z);
        s.w = fmaf(a, s.w, wx * bv.w);
        reinterpret_cast<float4 *>(hb + (int64_t)p * N)[lane] = s;
        float acc = s.x * cv.x + s.y * cv.y + s.z * cv.z + s.w * cv.w;
        acc = warp_sum(acc);
        if (lane == 0) yb[p] = from_f<T>(acc + Dh * xr);
    }
}

}  // namespace

ssd_status step_launch(const Problem &pr, float *h, const void *x, const void *dt,
                       const float *A, const void *B, const void *C, const float *D,
                       void *y, cudaStream_t st, const DtPre &pre) {
    const DtPreArgs pa{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    const int64_t blocks = pr.batch * pr.nheads;
    if (blocks == 0) return SSD_OK;
    const int H = (int)pr.nheads, P = (int)pr.headdim, N = (int)pr.dstate,
              G = (int)pr.ngroups;
    launch_begin("ssd_step", st);
    if (N == 128 && P == 64) {
        if (pr.dtype == SSD_F32)
            step_kernel_n128<float><<<(unsigned)blocks, kStepThreads, 0, st>>>(
                h, (const float *)x, (const float *)dt, A, (const float *)B, (const float *)C, D,
                (float *)y, H, G, pa);
        else
            step_kernel_n128<__nv_bfloat16><<<(unsigned)blocks, kStepThreads, 0, st>>>(
                h, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)dt, A,
                (const __nv_bfloat16 *)B, (const __nv_bfloat16 *)C, D, (__nv_bfloat16 *)y, H, G,
                pa);
    } else if (pr.dtype == SSD_F32) {
        step_kernel<float><<<(unsigned)blocks, kStepThreads, 0, st>>>(
            h, (const float *)x, (const float *)dt, A, (const float *)B, (const float *)C, D,
            (float *)y, H, P, N, G, pa);
    } else {
        using bf = __nv_bfloat16;
        step_kernel<bf><<<(unsigned)blocks, kStepThreads, 0, st>>>(
            h, (const bf *)x, (const bf *)dt, A, (const bf *)B, (const bf *)C, D, (bf *)y, H,
            P, N, G, pa);
    }
    launch_end(st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "ssd_step launch");
    return SSD_OK;
}

}  // namespace ssd
