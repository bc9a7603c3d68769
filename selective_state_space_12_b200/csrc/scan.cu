// Selective scan with a diagonal A per channel ("精读笔记 #12：Mamba",
// llm-papers-study, sections 2.2 and 3, algorithm 2): the prior art the SSD
// pages measure their chunked algorithm against. For batch b, channel d (of
// D; group g = d / (D/G)), state index n (of N), token t:
//
//   dt = prepared step of (b, t, d)   (step options: bias, softplus, clamp)
//   h[n] = exp(dt A[d][n]) h[n] + w[n] x[t][d] B[t][g][n]
//   y[t][d] = sum_n C[t][g][n] h[n] + Dskip[d] x[t][d]
//
// with w[n] = dt (Euler) or (exp(dt A[d][n]) - 1) / A[d][n] (zero-order
// hold). Every state entry takes its own exponential every token, so no
// matrix unit applies: the kernel is bound by the exponential (MUFU) and FMA
// pipes, not by HBM. N / 4 consecutive lanes share a (b, d) channel, each
// keeping 4 of its states, A[d][n] log2 e and (ZOH) 1 / A[d][n] in registers
// while walking the sequence (four times the warps of one thread per channel,
// to hide the FMA, exponential and load latencies); y is summed across them
// by shuffles. The next token's x, dt, B and C are loaded one trip ahead;
// B and C are the same for every channel of a group (cached lines).
#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

constexpr int kScanThreads = 128;
constexpr int kPer = 4;  // states per thread
constexpr float kLog2eS = 1.4426950408889634f;

// kPer consecutive elements of a B or C row as floats
template <typename T>
__device__ __forceinline__ float4 load_quad(const T *p) {
    return load4(p);
}

// TPC = N / kPer threads per channel (consecutive lanes of a warp), each
// holding kPer of the channel's states; y is summed across them by shuffles.
// (The staged kernel below takes the states per thread as a parameter.)
template <typename T, int N, bool ZOH>
__global__ void __launch_bounds__(kScanThreads)
selective_scan_kernel(const T *__restrict__ x, const T *__restrict__ dt,
                      const float *__restrict__ A, const T *__restrict__ B,
                      const T *__restrict__ C, const float *__restrict__ Dskip,
                      const float *__restrict__ h0, T *__restrict__ y,
                      float *__restrict__ h_final, int L, int D, int G, const DtPreArgs pre,
                      int pre_on) {
    constexpr int TPC = N / kPer;
    static_assert(N % kPer == 0 && TPC >= 1 && TPC <= 32 && (TPC & (TPC - 1)) == 0, "N");
    const int gt = blockIdx.x * kScanThreads + threadIdx.x;
    const int q = gt % TPC;  // which kPer states of the channel
    const int b = blockIdx.y;
    // lanes past the last channel run on a copy of it and store nothing, so
    // that every lane of the warp takes part in the shuffles
    const bool active = gt / TPC < D;
    const int d = active ? gt / TPC : D - 1;
    const int g = d / (D / G);
    const int n0 = q * kPer;
    const int64_t lane = (int64_t)b * D + d;
    // Ak: A (zero-order hold, which needs exp(dt A) - 1) or A log2 e (Euler,
    // one exp2 per entry)
    float h[kPer], Ak[kPer], invA[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const float a = A[(int64_t)d * N + n0 + k];
        Ak[k] = ZOH ? a : a * kLog2eS;
        invA[k] = (ZOH && a != 0.f) ? 1.f / a : 0.f;
        h[k] = h0 ? h0[lane * N + n0 + k] : 0.f;
    }
    const float bias = (pre_on && pre.bias) ? pre.bias[d] : 0.f;
    const float Dd = Dskip ? Dskip[d] : 0.f;
    const int64_t step_x = D, step_bc = (int64_t)G * N;
    const T *xp = x + (int64_t)b * L * D + d;
    const T *dp = dt + (int64_t)b * L * D + d;
    const T *Bp = B + ((int64_t)b * L * G + g) * N + n0;
    const T *Cp = C + ((int64_t)b * L * G + g) * N + n0;
    T *yp = y + (int64_t)b * L * D + d;
    // one trip ahead
    float xn = 0.f, dn = 0.f;
    float4 Bn = make_float4(0.f, 0.f, 0.f, 0.f), Cn = Bn;
    if (L > 0) {
        xn = to_f(xp[0]);
        dn = to_f(dp[0]);
        Bn = load_quad(Bp);
        Cn = load_quad(Cp);
    }
#pragma unroll 1
    for (int t = 0; t < L; ++t) {
        const float xv = xn, raw = dn;
        const float Bt[kPer] = {Bn.x, Bn.y, Bn.z, Bn.w};
        const float Ct[kPer] = {Cn.x, Cn.y, Cn.z, Cn.w};
        if (t + 1 < L) {
            xn = to_f(xp[(int64_t)(t + 1) * step_x]);
            dn = to_f(dp[(int64_t)(t + 1) * step_x]);
            Bn = load_quad(Bp + (int64_t)(t + 1) * step_bc);
            Cn = load_quad(Cp + (int64_t)(t + 1) * step_bc);
        }
        // bf16 I/O takes the compact softplus (relative error below 3e-5)
        const float dtv = !pre_on ? raw
                          : (sizeof(T) == 2 ? prepare_dt_compact(raw, bias, pre)
                                            : prepare_dt(raw, bias, pre));
        const float u = dtv * xv;  // Euler: input weight dt times x
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            float a, wx;
            if (ZOH) {
                // exp(dt A) - 1 without cancellation (compact expm1), the
                // decay from it, and the hold weight (exp(dt A) - 1) / A
                const float em1 = expm1_compact(dtv * Ak[k]);
                a = em1 + 1.f;
                wx = (Ak[k] != 0.f) ? em1 * invA[k] * xv : u;
            } else {
                a = tc::fast_exp2(dtv * Ak[k]);
                wx = u;
            }
            h[k] = fmaf(a, h[k], wx * Bt[k]);
            acc = fmaf(Ct[k], h[k], acc);
        }
#pragma unroll
        for (int o = 1; o < TPC; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (q == 0 && active) yp[(int64_t)t * step_x] = from_f<T>(fmaf(Dd, xv, acc));
    }
    if (h_final && active) {
#pragma unroll
        for (int k = 0; k < kPer; ++k) h_final[lane * N + n0 + k] = h[k];
    }
}

// States per thread in the staged kernel (the per-lane kernel keeps kPer):
// eight, so that each token's per-thread work (x, dt and the B, C rows from
// shared memory, the shuffle that sums y, the store) is shared by eight state
// updates; measured on the 2.8B-style scan: 4 per thread 1006 us, 8 886 us,
// 16 943 us (too few warps per SM).
#ifndef SSD_SCAN_PER
#define SSD_SCAN_PER 8
#endif
constexpr int kStagedPer = SSD_SCAN_PER;
// Tokens per trip of the staged loop: sixteen, so that the exponentials of
// the next tokens are in flight while one token's state updates wait on theirs
// (8 states per thread, scalar update: 887 us with one, 843 with two, 810
// with four, 799 with eight; packed pairs, 64-thread blocks: 721 with four,
// 720 with eight, 713 with sixteen).
#ifndef SSD_SCAN_UNROLL
#define SSD_SCAN_UNROLL 16
#endif
constexpr int kScanUnroll = SSD_SCAN_UNROLL;
// Threads per block of the staged kernel: 64 (32 channels of N = 16), 720 us
// against 732 with 128 and 749 with 32 on the 2.8B-style scan.
#ifndef SSD_SCAN_THREADS
#define SSD_SCAN_THREADS 64
#endif
constexpr int kStagedThreads = SSD_SCAN_THREADS;

using tc::f2;
using tc::f2_fma;
using tc::f2_mul;
using tc::f2_pack;
using tc::f2_sub;
using tc::f2_unpack;

// The same recurrence with the block's inputs staged in shared memory: TT
// tokens at a time of x and dt for the block's channels and of B and C for
// its group, by asynchronous 16-byte copies, double-buffered (chunk c + 1
// lands while chunk c is computed). Needs 16-byte rows: D a multiple of
// 16 / sizeof(T), and all of a block's channels in one group. TT keeps a
// chunk's x or dt tile at 2 KB (16 to 64 tokens): about 20 KB of shared
// memory for a 64-thread block of bf16 N = 16, so that the ~9 blocks an SM
// gets on the 2.8B-style scan are all resident at once.
#ifndef SSD_SCAN_TILE_BYTES
#define SSD_SCAN_TILE_BYTES 2048
#endif
template <typename T, int CPB>
__host__ __device__ constexpr int chunk_tokens() {
    constexpr int t = SSD_SCAN_TILE_BYTES / (CPB * (int)sizeof(T));
    return t > 64 ? 64 : (t < 16 ? 16 : t);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool full) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    const int n = full ? 16 : 0;  // 0: zero fill, nothing read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int K>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory");
}

template <typename T, int N, int PER, bool ZOH>
__global__ void __launch_bounds__(kStagedThreads)
selective_scan_staged(const T *__restrict__ x, const T *__restrict__ dt,
                      const float *__restrict__ A, const T *__restrict__ B,
                      const T *__restrict__ C, const float *__restrict__ Dskip,
                      const float *__restrict__ h0, T *__restrict__ y,
                      float *__restrict__ h_final, int L, int D, int G, const DtPreArgs pre,
                      int pre_on) {
    constexpr int TPC = N / PER;
    constexpr int CPB = kStagedThreads / TPC;     // channels per block
    constexpr int EPP = 16 / sizeof(T);         // elements per 16-byte piece
    constexpr int XP = CPB / EPP;               // pieces per x / dt row
    constexpr int BP = (N + EPP - 1) / EPP;     // pieces per B / C row
    static_assert(CPB % EPP == 0 && (N * sizeof(T)) % 16 == 0, "16-byte rows");
    constexpr int kTT = chunk_tokens<T, CPB>();
    static_assert(PER % 2 == 0, "states are updated in pairs");
    __shared__ __align__(16) T sx[2][kTT][CPB];
    __shared__ __align__(16) T sdt[2][kTT][CPB];
    __shared__ __align__(16) T sB[2][kTT][N];
    __shared__ __align__(16) T sC[2][kTT][N];
    __shared__ float sdtp[kTT][CPB];  // the chunk's prepared steps
    __shared__ __align__(16) float sBf[kTT][N], sCf[kTT][N];  // its B, C rows as floats
    __shared__ float sbias[CPB];
    const int tid = threadIdx.x;
    const int c = tid / TPC, q = tid % TPC;     // channel within the block, state quarter
    const int d0 = blockIdx.x * CPB;
    const int b = blockIdx.y;
    const bool active = d0 + c < D;
    const int d = active ? d0 + c : D - 1;
    const int g = d0 / (D / G);                 // one group per block
    const int n0 = q * PER;
    const int64_t lane = (int64_t)b * D + d;
    float h[PER], Ak[PER], invA[PER], Ak2[PER];
    bool nonzero_A = true;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const float a = A[(int64_t)d * N + n0 + k];
        Ak[k] = ZOH ? a : a * kLog2eS;
        Ak2[k] = a * kLog2eS;
        invA[k] = (ZOH && a != 0.f) ? 1.f / a : 0.f;
        nonzero_A = nonzero_A && a != 0.f;
        h[k] = h0 ? h0[lane * N + n0 + k] : 0.f;
    }
    // bf16 I/O, zero-order hold, A != 0 throughout: h <- e h + (e - 1) c with
    // e = exp(dt A) from one exp2 and c = (x / A) B, taken as e (h + c) - c
    // (its cancellation, ~1e-7 / |dt A| relative, only where the input term is
    // negligible for bf16)
    const bool lean = ZOH && sizeof(T) == 2 && nonzero_A;
    for (int i = tid; i < CPB; i += kStagedThreads)
        sbias[i] = (pre_on && pre.bias && d0 + i < D) ? pre.bias[d0 + i] : 0.f;
    const float Dd = Dskip ? Dskip[d] : 0.f;
    const T *xb = x + (int64_t)b * L * D;
    const T *db = dt + (int64_t)b * L * D;
    const T *Bb = B + ((int64_t)b * L * G + g) * N;
    const T *Cb = C + ((int64_t)b * L * G + g) * N;
    T *yp = y + (int64_t)b * L * D + d;
    const int nchunks = (L + kTT - 1) / kTT;
    // the pieces of one chunk: x and dt rows (XP each), B and C rows (BP each)
    auto stage = [&](int buf, int t0) {
        for (int i = tid; i < kTT * XP; i += kStagedThreads) {
            const int r = i / XP, p = i % XP;
            const int t = t0 + r, ch = d0 + p * EPP;
            const bool ok = t < L && ch < D;
            const int64_t off = (int64_t)(ok ? t : 0) * D + (ok ? ch : 0);
            cp_async16(&sx[buf][r][p * EPP], xb + off, ok);
            cp_async16(&sdt[buf][r][p * EPP], db + off, ok);
        }
        for (int i = tid; i < kTT * BP; i += kStagedThreads) {
            const int r = i / BP, p = i % BP;
            const int t = t0 + r;
            const bool ok = t < L;
            const int64_t off = (int64_t)(ok ? t : 0) * G * N + p * EPP;
            cp_async16(&sB[buf][r][p * EPP], Bb + off, ok);
            cp_async16(&sC[buf][r][p * EPP], Cb + off, ok);
        }
        cp_async_commit();
    };
    if (nchunks > 0) stage(0, 0);
#pragma unroll 1
    for (int ci = 0; ci < nchunks; ++ci) {
        const int buf = ci & 1, t0 = ci * kTT;
        if (ci + 1 < nchunks) {
            stage(buf ^ 1, t0 + kTT);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int tn = min(kTT, L - t0);
        // each step prepared once (not once per state quarter); bf16 I/O takes
        // the compact softplus (relative error below 3e-5)
        for (int i = tid; i < tn * CPB; i += kStagedThreads) {
            const int r = i / CPB, cc = i % CPB;
            const float raw = to_f(sdt[buf][r][cc]);
            sdtp[r][cc] = !pre_on ? raw
                          : (sizeof(T) == 2 ? prepare_dt_compact(raw, sbias[cc], pre)
                                            : prepare_dt(raw, sbias[cc], pre));
        }
        // B and C converted once per chunk, not once per lane and token
        for (int i = tid; i < tn * N; i += kStagedThreads) {
            const int r = i / N, n = i % N;
            sBf[r][n] = to_f(sB[buf][r][n]);
            sCf[r][n] = to_f(sC[buf][r][n]);
        }
        __syncthreads();
#pragma unroll kScanUnroll
        for (int r = 0; r < tn; ++r) {
            const float xv = to_f(sx[buf][r][c]);
            const float dtv = sdtp[r][c];
            float Bt[PER], Ct[PER];
#pragma unroll
            for (int k4 = 0; k4 < PER / 4; ++k4) {
                const float4 Bq = *reinterpret_cast<const float4 *>(&sBf[r][n0 + 4 * k4]);
                const float4 Cq = *reinterpret_cast<const float4 *>(&sCf[r][n0 + 4 * k4]);
                Bt[4 * k4] = Bq.x; Bt[4 * k4 + 1] = Bq.y; Bt[4 * k4 + 2] = Bq.z; Bt[4 * k4 + 3] = Bq.w;
                Ct[4 * k4] = Cq.x; Ct[4 * k4 + 1] = Cq.y; Ct[4 * k4 + 2] = Cq.z; Ct[4 * k4 + 3] = Cq.w;
            }
            const float u = dtv * xv;
            float acc = 0.f;
            if (lean) {
                // pairs of states in packed fp32 arithmetic: h <- e (h + c) - c,
                // with -c = (x / A)(-1) B exact, one rounding more than
                // e h + (e c - c) (scalar update 802 us, packed 732)
                const f2 dt2 = f2_pack(dtv, dtv), nx2 = f2_pack(-xv, -xv);
                f2 acc2 = f2_pack(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < PER; k += 2) {
                    float a0, a1;
                    f2_unpack(f2_mul(dt2, f2_pack(Ak2[k], Ak2[k + 1])), a0, a1);
                    const f2 e2 = f2_pack(tc::fast_exp2(a0), tc::fast_exp2(a1));
                    const f2 ncb = f2_mul(f2_mul(f2_pack(invA[k], invA[k + 1]), nx2),
                                          f2_pack(Bt[k], Bt[k + 1]));
                    const f2 hn = f2_fma(e2, f2_sub(f2_pack(h[k], h[k + 1]), ncb), ncb);
                    f2_unpack(hn, h[k], h[k + 1]);
                    acc2 = f2_fma(f2_pack(Ct[k], Ct[k + 1]), hn, acc2);
                }
                float s0, s1;
                f2_unpack(acc2, s0, s1);
                acc = s0 + s1;
            } else {
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                float a, wx;
                if (ZOH) {
                    // bf16 I/O: exp(dt A) - 1 from one hardware exp (its
                    // cancellation, ~6e-8 / |dt A| relative, only where the
                    // input term is negligible); fp32: the compact expm1
                    const float xa = dtv * Ak[k];
                    const float em1 = sizeof(T) == 2 ? tc::fast_exp2(xa * kLog2eS) - 1.f
                                                     : expm1_compact(xa);
                    a = em1 + 1.f;
                    wx = (Ak[k] != 0.f) ? em1 * invA[k] * xv : u;
                } else {
                    a = tc::fast_exp2(dtv * Ak[k]);
                    wx = u;
                }
                h[k] = fmaf(a, h[k], wx * Bt[k]);
                acc = fmaf(Ct[k], h[k], acc);
            }
            }
#pragma unroll
            for (int o = 1; o < TPC; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (q == 0 && active) yp[(int64_t)(t0 + r) * D] = from_f<T>(fmaf(Dd, xv, acc));
        }
        __syncthreads();  // the buffer is refilled two chunks later
    }
    if (h_final && active) {
#pragma unroll
        for (int k = 0; k < PER; ++k) h_final[lane * N + n0 + k] = h[k];
    }
}



template <typename T, int N>
cudaError_t launch_scan_t(const Problem &pr, const void *x, const void *dt, const float *A,
                          const void *B, const void *C, const float *Dskip, const float *h0,
                          void *y, float *h_final, const DtPre &pre, cudaStream_t st) {
    const int D = (int)pr.nheads;
    constexpr int TPC = N / kPer;
    const long long threads = (long long)D * TPC;
    dim3 grid((unsigned)((threads + kScanThreads - 1) / kScanThreads), (unsigned)pr.batch);
    const DtPreArgs pa{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    const int pre_on = (pre.bias || pre.softplus || pre.dt_max > 0.f) ? 1 : 0;
    constexpr int SPER = kStagedPer < N ? kStagedPer : N;
    constexpr int CPB = kStagedThreads / (N / SPER);
    constexpr bool kStageable = (CPB % (int)(16 / sizeof(T)) == 0) && (N * sizeof(T)) % 16 == 0;
    launch_begin("selective_scan", st);
    if constexpr (kStageable) {
        const bool staged = (D % (int)(16 / sizeof(T)) == 0) &&
                            (pr.ngroups == 1 || (D / pr.ngroups) % CPB == 0);
        if (staged) {
            dim3 sgrid((unsigned)((D + CPB - 1) / CPB), (unsigned)pr.batch);
            if (pre.zoh)
                selective_scan_staged<T, N, SPER, true><<<sgrid, kStagedThreads, 0, st>>>(
                    (const T *)x, (const T *)dt, A, (const T *)B, (const T *)C, Dskip, h0,
                    (T *)y, h_final, (int)pr.seqlen, D, (int)pr.ngroups, pa, pre_on);
            else
                selective_scan_staged<T, N, SPER, false><<<sgrid, kStagedThreads, 0, st>>>(
                    (const T *)x, (const T *)dt, A, (const T *)B, (const T *)C, Dskip, h0,
                    (T *)y, h_final, (int)pr.seqlen, D, (int)pr.ngroups, pa, pre_on);
            launch_end(st);
            return cudaGetLastError();
        }
    }
    if (pre.zoh)
        selective_scan_kernel<T, N, true><<<grid, kScanThreads, 0, st>>>(
            (const T *)x, (const T *)dt, A, (const T *)B, (const T *)C, Dskip, h0, (T *)y,
            h_final, (int)pr.seqlen, D, (int)pr.ngroups, pa, pre_on);
    else
        selective_scan_kernel<T, N, false><<<grid, kScanThreads, 0, st>>>(
            (const T *)x, (const T *)dt, A, (const T *)B, (const T *)C, Dskip, h0, (T *)y,
            h_final, (int)pr.seqlen, D, (int)pr.ngroups, pa, pre_on);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_scan_n(const Problem &pr, const void *x, const void *dt, const float *A,
                          const void *B, const void *C, const float *Dskip, const float *h0,
                          void *y, float *h_final, const DtPre &pre, cudaStream_t st) {
    switch (pr.dstate) {
        case 4: return launch_scan_t<T, 4>(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre, st);
        case 8: return launch_scan_t<T, 8>(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre, st);
        default: return launch_scan_t<T, 16>(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre, st);
    }
}

}  // namespace

bool scan_supported_dstate(int64_t N) { return N == 4 || N == 8 || N == 16; }

ssd_status scan_launch(const Problem &pr, const void *x, const void *dt, const float *A,
                       const void *B, const void *C, const float *Dskip, const float *h0,
                       void *y, float *h_final, const DtPre &pre, cudaStream_t st) {
    if (pr.batch * pr.nheads == 0) return SSD_OK;
    const cudaError_t e =
        pr.dtype == SSD_F32
            ? launch_scan_n<float>(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre, st)
            : launch_scan_n<__nv_bfloat16>(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre, st);
    if (e != cudaSuccess) return cuda_fail(e, "selective_scan launch");
    return SSD_OK;
}

}  // namespace ssd
