// General forward path on CUDA cores (fp32 FMA), for fp32 or bf16 I/O and
// every supported size. The chunked algorithm in three launches
// ("Mamba-2 — 注意力的远亲", section "两条路各走一半"; "Mamba-2 模型解读",
// sections 6.1-6.2):
//
//   1. chunk_state  — per (b, h, chunk): the within-chunk cumulative
//      log-decay cum_j = sum_{k<=j} dt_k A_h (the segsum's running sum), the
//      chunk's total decay exp(cum_end), and its own state
//      S_c = sum_j exp(cum_end - cum_j) w_j x_j (x) B_j   (input -> state),
//      w_j the input weight: dt_j, or the zero-order hold under the step
//      options (common.cuh: prepare_dt, input_weight).
//   2. state_pass   — per (b, h, p, n): H_0 = h0, H_{c+1} = exp(cum_end,c) H_c
//      + S_c, written over S_c in place; h_final = H_nc   (state -> state).
//   3. chunk_output — per (b, h, chunk, 64-row tile): the diagonal block
//      (L o C B^T)(w x) with L_ij = exp(cum_i - cum_j) for j <= i, plus
//      exp(cum_i) C_i . H_c (state -> output), plus D x.
//
// fp32 I/O runs this path (no tensor-core type reaches fp32 accuracy); the
// tensor-core path serves bf16.
#include <stdio.h>

#include "common.cuh"
#include "internal.h"

namespace ssd {
namespace {

constexpr int kThreads = 256;  // also the largest chunk: one token per thread

// ADJ (backward pass): the same contraction with weight exp(cum_i) on (dy, C)
// instead of exp(cum_end - cum_j) w_j on (x, B): each chunk's contribution
// sum_i exp(cum_i) dy_i (x) C_i to the gradient of its entering state.
template <typename T, bool ADJ = false>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(const T *__restrict__ x, const T *__restrict__ dt,
                   const float *__restrict__ A, const T *__restrict__ B,
                   float *__restrict__ S, float *__restrict__ decay, int L, int H,
                   int P, int N, int G, int Q, int nc, const DtPreArgs pre) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q;
    const int len = min(Q, L - t0);
    const int tid = threadIdx.x;
    __shared__ float s_w[kThreads];
    __shared__ float s_tot[32];
    __shared__ float s_total;
    __shared__ float xs[32][65];
    __shared__ float bs[32][65];

    float wj = 0.f, ell = 0.f;
    if (tid < len) {
        const float dtj = prepare_dt(to_f(dt[((int64_t)b * L + t0 + tid) * H + h]), h, pre);
        ell = dtj * A[h];
        wj = input_weight(dtj, A[h], pre.zoh);
    }
    const float cum = block_inclusive_scan(ell, s_tot);
    if (tid == len - 1) s_total = cum;
    __syncthreads();
    const float total = s_total;
    if (tid < len) s_w[tid] = ADJ ? expf(cum) : expf(total - cum) * wj;
    if (tid == 0) decay[((int64_t)b * H + h) * nc + c] = expf(total);
    __syncthreads();

    const int tx = tid & 15, ty = tid >> 4;
    const int64_t row0 = (int64_t)b * L + t0;
    float *Sp = S + (((int64_t)b * H + h) * nc + c) * (int64_t)P * N;
    for (int p0 = 0; p0 < P; p0 += 64) {
        for (int n0 = 0; n0 < N; n0 += 64) {
            float acc[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[r][k] = 0.f;
            for (int j0 = 0; j0 < len; j0 += 32) {
                for (int idx = tid; idx < 32 * 64; idx += kThreads) {
                    const int jj = idx >> 6, cc = idx & 63, j = j0 + jj;
                    float xv = 0.f, bv = 0.f;
                    if (j < len) {
                        if (p0 + cc < P)
                            xv = s_w[j] * to_f(x[((row0 + j) * H + h) * P + p0 + cc]);
                        if (n0 + cc < N) bv = to_f(B[((row0 + j) * G + g) * N + n0 + cc]);
                    }
                    xs[jj][cc] = xv;
                    bs[jj][cc] = bv;
                }
                __syncthreads();
#pragma unroll 8
                for (int jj = 0; jj < 32; ++jj) {
                    float av[4], bv[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) av[r] = xs[jj][ty + 16 * r];
#pragma unroll
                    for (int k = 0; k < 4; ++k) bv[k] = bs[jj][tx + 16 * k];
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int k = 0; k < 4; ++k) acc[r][k] = fmaf(av[r], bv[k], acc[r][k]);
                }
                __syncthreads();
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int p = p0 + ty + 16 * r, n = n0 + tx + 16 * k;
                    if (p < P && n < N) Sp[(int64_t)p * N + n] = acc[r][k];
                }
        }
    }
}

// One thread per 4 consecutive state entries of one (b, h); sequential over
// chunks. S holds each chunk's own state on entry and the state entering each
// chunk on exit. decay_total (nullable) receives the product of the chunks'
// decays: the total decay of the lane's sequence.
__global__ void __launch_bounds__(kThreads)
state_pass_kernel(float *__restrict__ S, const float *__restrict__ decay,
                  const float *h0, float *h_final, int H, int PN4, int nc,
                  float *decay_total) {
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (q >= PN4) return;
    const int64_t lane = (int64_t)b * H + h;
    float4 st = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h0) st = reinterpret_cast<const float4 *>(h0 + lane * PN4 * 4)[q];
    float4 *Sp = reinterpret_cast<float4 *>(S + lane * nc * (int64_t)PN4 * 4);
    const float *dp = decay + lane * nc;
    float4 s_next = make_float4(0.f, 0.f, 0.f, 0.f);
    if (nc > 0) s_next = Sp[q];
    float dprod = 1.f;
    for (int c = 0; c < nc; ++c) {
        const float4 s = s_next;
        if (c + 1 < nc) s_next = Sp[(int64_t)(c + 1) * PN4 + q];
        const float d = dp[c];
        dprod *= d;
        Sp[(int64_t)c * PN4 + q] = st;
        st.x = fmaf(d, st.x, s.x);
        st.y = fmaf(d, st.y, s.y);
        st.z = fmaf(d, st.z, s.z);
        st.w = fmaf(d, st.w, s.w);
    }
    if (h_final) reinterpret_cast<float4 *>(h_final + lane * PN4 * 4)[q] = st;
    if (decay_total && q == 0) decay_total[lane] = dprod;
}

// Sequence parallelism: the state entering piece `part` of a sequence split
// into `nparts` consecutive pieces, from each piece's own end state (from a
// zero initial state) and total decay: h_in = h0, then for r < part
// h_in <- decay_r h_in + S_r ("两条路各走一半": only the block-end state
// passes between blocks). h_total (nullable) receives the chain over all
// pieces, the whole sequence's final state. S (nparts, lanes, P*N),
// decays (nparts, lanes).
__global__ void __launch_bounds__(kThreads)
state_chain_kernel(const float *__restrict__ S, const float *__restrict__ decays,
                   const float *h0, float *h_in, float *h_total, int64_t lanes, int PN4,
                   int nparts, int part) {
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lane = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
    if (q >= PN4 || lane >= lanes) return;
    float4 st = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h0) st = reinterpret_cast<const float4 *>(h0 + lane * PN4 * 4)[q];
    const int last = h_total ? nparts : part;
    for (int r = 0; r < last; ++r) {
        if (r == part && h_in) reinterpret_cast<float4 *>(h_in + lane * PN4 * 4)[q] = st;
        const float d = decays[(int64_t)r * lanes + lane];
        const float4 s = reinterpret_cast<const float4 *>(S + ((int64_t)r * lanes + lane) * PN4 * 4)[q];
        st.x = fmaf(d, st.x, s.x);
        st.y = fmaf(d, st.y, s.y);
        st.z = fmaf(d, st.z, s.z);
        st.w = fmaf(d, st.w, s.w);
    }
    if (part >= last && h_in) reinterpret_cast<float4 *>(h_in + lane * PN4 * 4)[q] = st;
    if (h_total) reinterpret_cast<float4 *>(h_total + lane * PN4 * 4)[q] = st;
}

struct OutSmem {
    int cum, dt, tot, Cf, Bs, Ws, XH, total;  // float offsets
};
__host__ __device__ inline OutSmem out_smem(int P, int N) {
    OutSmem s;
    s.cum = 0;
    s.dt = 256;
    s.tot = 512;
    s.Cf = 544;
    s.Bs = s.Cf + 64 * (N + 1);
    s.Ws = s.Bs + 64 * 65;
    s.XH = s.Ws + 64 * 65;
    const int xh = (P * 65 > 64 * (P + 1)) ? P * 65 : 64 * (P + 1);
    s.total = s.XH + xh;
    return s;
}

// RP = P / 16 output columns per thread.
template <typename T, int RP>
__global__ void __launch_bounds__(kThreads)
chunk_output_kernel(const T *__restrict__ x, const T *__restrict__ dt,
                    const float *__restrict__ A, const T *__restrict__ B,
                    const T *__restrict__ C, const float *__restrict__ D,
                    const float *__restrict__ Hst, T *__restrict__ y, int L, int H, int N,
                    int G, int Q, int nc, int ntile, const DtPreArgs pre) {
    constexpr int P = RP * 16;
    const int c = blockIdx.x / ntile, it = blockIdx.x % ntile;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q;
    const int len = min(Q, L - t0);
    const int i0 = it * 64;
    if (i0 >= len) return;  // uniform over the block, before any barrier
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    extern __shared__ float smem[];
    const OutSmem lay = out_smem(P, N);
    float *s_cum = smem + lay.cum;
    float *s_dt = smem + lay.dt;
    float *s_tot = smem + lay.tot;
    float *Cf = smem + lay.Cf;  // [64][N+1]
    float *Bs = smem + lay.Bs;  // [64][65]
    float *Ws = smem + lay.Ws;  // [64][65]
    float *XH = smem + lay.XH;  // H slice [P][65], then x tile [64][P+1]
    const int64_t row0 = (int64_t)b * L + t0;

    float wj = 0.f, ell = 0.f;  // input weight and log-decay of token tid
    if (tid < len) {
        const float dtj = prepare_dt(to_f(dt[(row0 + tid) * H + h]), h, pre);
        ell = dtj * A[h];
        wj = input_weight(dtj, A[h], pre.zoh);
    }
    const float cum = block_inclusive_scan(ell, s_tot);
    s_cum[tid] = cum;
    s_dt[tid] = wj;
    for (int idx = tid; idx < 64 * N; idx += kThreads) {
        const int ii = idx / N, n = idx - ii * N, i = i0 + ii;
        Cf[ii * (N + 1) + n] = (i < len) ? to_f(C[((row0 + i) * G + g) * N + n]) : 0.f;
    }
    __syncthreads();

    // state -> output: accO[i][p] = sum_n C_i[n] H_c[p][n]
    float accO[4][RP], accD[4][RP];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int k = 0; k < RP; ++k) accO[r][k] = accD[r][k] = 0.f;
    const float *Hc = Hst + (((int64_t)b * H + h) * nc + c) * (int64_t)P * N;
    for (int n0 = 0; n0 < N; n0 += 64) {
        for (int idx = tid; idx < P * 64; idx += kThreads) {
            const int pp = idx >> 6, nn = idx & 63;
            XH[pp * 65 + nn] = (n0 + nn < N) ? Hc[(int64_t)pp * N + n0 + nn] : 0.f;
        }
        __syncthreads();
        const int nlim = min(64, N - n0);
        for (int nn = 0; nn < nlim; ++nn) {
            float cv[4], hv[RP];
#pragma unroll
            for (int r = 0; r < 4; ++r) cv[r] = Cf[(ty + 16 * r) * (N + 1) + n0 + nn];
#pragma unroll
            for (int k = 0; k < RP; ++k) hv[k] = XH[(tx + 16 * k) * 65 + nn];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < RP; ++k) accO[r][k] = fmaf(cv[r], hv[k], accO[r][k]);
        }
        __syncthreads();
    }

    // diagonal block: accD[i][p] = sum_{j<=i} exp(cum_i - cum_j) dt_j (C_i.B_j) x_j[p]
    for (int jt = 0; jt <= it; ++jt) {
        const int j0 = jt * 64;
        float G4[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int k = 0; k < 4; ++k) G4[r][k] = 0.f;
        for (int n0 = 0; n0 < N; n0 += 64) {
            for (int idx = tid; idx < 64 * 64; idx += kThreads) {
                const int jj = idx >> 6, nn = idx & 63, j = j0 + jj;
                Bs[jj * 65 + nn] = (j < len && n0 + nn < N)
                                       ? to_f(B[((row0 + j) * G + g) * N + n0 + nn])
                                       : 0.f;
            }
            __syncthreads();
            const int nlim = min(64, N - n0);
            for (int nn = 0; nn < nlim; ++nn) {
                float cv[4], bv[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) cv[r] = Cf[(ty + 16 * r) * (N + 1) + n0 + nn];
#pragma unroll
                for (int k = 0; k < 4; ++k) bv[k] = Bs[(tx + 16 * k) * 65 + nn];
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int k = 0; k < 4; ++k) G4[r][k] = fmaf(cv[r], bv[k], G4[r][k]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + ty + 16 * r, j = j0 + tx + 16 * k;
                float wv = 0.f;
                if (j <= i && i < len) wv = G4[r][k] * expf(s_cum[i] - s_cum[j]) * s_dt[j];
                Ws[(ty + 16 * r) * 65 + tx + 16 * k] = wv;
            }
        for (int idx = tid; idx < 64 * P; idx += kThreads) {
            const int jj = idx / P, pp = idx - jj * P, j = j0 + jj;
            XH[jj * (P + 1) + pp] = (j < len) ? to_f(x[((row0 + j) * H + h) * P + pp]) : 0.f;
        }
        __syncthreads();
        for (int jj = 0; jj < 64; ++jj) {
            float wv[4], xv[RP];
#pragma unroll
            for (int r = 0; r < 4; ++r) wv[r] = Ws[(ty + 16 * r) * 65 + jj];
#pragma unroll
            for (int k = 0; k < RP; ++k) xv[k] = XH[jj * (P + 1) + tx + 16 * k];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < RP; ++k) accD[r][k] = fmaf(wv[r], xv[k], accD[r][k]);
        }
        __syncthreads();
    }

    // epilogue: the last x tile loaded is this block's own rows (jt == it)
    const float Dh = D ? D[h] : 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int ii = ty + 16 * r, i = i0 + ii;
        if (i >= len) continue;
        const float e = expf(s_cum[i]);
#pragma unroll
        for (int k = 0; k < RP; ++k) {
            const int p = tx + 16 * k;
            const float xv = XH[ii * (P + 1) + p];
            const float v = accD[r][k] + e * accO[r][k] + Dh * xv;
            y[((row0 + i) * H + h) * P + p] = from_f<T>(v);
        }
    }
}

template <typename T, int RP>
cudaError_t launch_output(const Problem &pr, const T *x, const T *dt, const float *A,
                          const T *B, const T *C, const float *D, const float *Hst, T *y,
                          cudaStream_t st, const DtPreArgs &pre) {
    const int nc = (int)pr.nchunks();
    const int ntile = (pr.chunk + 63) / 64;
    const OutSmem lay = out_smem(RP * 16, (int)pr.dstate);
    const size_t smem = (size_t)lay.total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(chunk_output_kernel<T, RP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(nc * ntile), (unsigned)pr.nheads, (unsigned)pr.batch);
    launch_begin("simt_chunk_output", st);
    chunk_output_kernel<T, RP><<<grid, kThreads, smem, st>>>(
        x, dt, A, B, C, D, Hst, y, (int)pr.seqlen, (int)pr.nheads, (int)pr.dstate,
        (int)pr.ngroups, pr.chunk, nc, ntile, pre);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T>
ssd_status forward_t(const Problem &pr, const T *x, const T *dt, const float *A, const T *B,
                     const T *C, const float *D, const float *h0, T *y, float *h_final,
                     void *ws, cudaStream_t st, const DtPreArgs &pre,
                     float *decay_total = nullptr, bool state_only = false) {
    const int nc = (int)pr.nchunks();
    const int64_t lanes = pr.batch * pr.nheads;
    float *S = static_cast<float *>(ws);
    float *decay = reinterpret_cast<float *>(
        static_cast<char *>(ws) + align256((size_t)lanes * nc * pr.headdim * pr.dstate * 4));
    cudaError_t e;
    if (nc > 0) {
        dim3 grid((unsigned)nc, (unsigned)pr.nheads, (unsigned)pr.batch);
        launch_begin("simt_chunk_state", st);
        chunk_state_kernel<T><<<grid, kThreads, 0, st>>>(
            x, dt, A, B, S, decay, (int)pr.seqlen, (int)pr.nheads, (int)pr.headdim,
            (int)pr.dstate, (int)pr.ngroups, pr.chunk, nc, pre);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "chunk_state launch");
    }
    {
        const int PN4 = (int)(pr.headdim * pr.dstate / 4);
        dim3 grid((unsigned)((PN4 + kThreads - 1) / kThreads), (unsigned)pr.nheads,
                  (unsigned)pr.batch);
        launch_begin("simt_state_pass", st);
        state_pass_kernel<<<grid, kThreads, 0, st>>>(S, decay, h0, h_final, (int)pr.nheads,
                                                     PN4, nc, decay_total);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "state_pass launch");
    }
    if (nc == 0 || state_only) return SSD_OK;
    switch (pr.headdim / 16) {
        case 1: e = launch_output<T, 1>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 2: e = launch_output<T, 2>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 3: e = launch_output<T, 3>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 4: e = launch_output<T, 4>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 5: e = launch_output<T, 5>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 6: e = launch_output<T, 6>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 7: e = launch_output<T, 7>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        case 8: e = launch_output<T, 8>(pr, x, dt, A, B, C, D, S, y, st, pre); break;
        default: return fail(SSD_ERR_UNSUPPORTED, "headdim %lld", (long long)pr.headdim);
    }
    if (e != cudaSuccess) return cuda_fail(e, "chunk_output launch");
    return SSD_OK;
}

}  // namespace

ssd_status state_pass_launch(float *S, const float *decay, const float *h0, float *h_final,
                             int64_t batch, int64_t nheads, int PN4, int nc, cudaStream_t st,
                             float *decay_total) {
    dim3 grid((unsigned)((PN4 + kThreads - 1) / kThreads), (unsigned)nheads, (unsigned)batch);
    launch_begin("state_pass", st);
    state_pass_kernel<<<grid, kThreads, 0, st>>>(S, decay, h0, h_final, (int)nheads, PN4, nc,
                                                 decay_total);
    launch_end(st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "state_pass launch");
    return SSD_OK;
}

size_t simt_workspace_bytes(const Problem &pr) {
    const size_t lanes = (size_t)(pr.batch * pr.nheads);
    const size_t nc = (size_t)pr.nchunks();
    return align256(lanes * nc * (size_t)(pr.headdim * pr.dstate) * 4) + align256(lanes * nc * 4);
}

ssd_status simt_state(const Problem &pr, const void *x, const void *dt, const float *A,
                      const void *B, float *state_out, float *decay_out, void *ws,
                      cudaStream_t st, const DtPre &pre) {
    const DtPreArgs pa{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    if (pr.dtype == SSD_F32)
        return forward_t<float>(pr, (const float *)x, (const float *)dt, A, (const float *)B,
                                nullptr, nullptr, nullptr, nullptr, state_out, ws, st, pa,
                                decay_out, true);
    using bf = __nv_bfloat16;
    return forward_t<bf>(pr, (const bf *)x, (const bf *)dt, A, (const bf *)B, nullptr, nullptr,
                         nullptr, nullptr, state_out, ws, st, pa, decay_out, true);
}

ssd_status chunk_states_launch(const Problem &pr, const void *x, const void *dt, const float *A,
                               const void *B, float *S, float *decay, bool adjoint,
                               cudaStream_t st) {
    const int nc = (int)pr.nchunks();
    if (nc == 0) return SSD_OK;
    dim3 grid((unsigned)nc, (unsigned)pr.nheads, (unsigned)pr.batch);
    const DtPreArgs pa{nullptr, 0, 0, 0.f, 0.f};
    const int L = (int)pr.seqlen, H = (int)pr.nheads, P = (int)pr.headdim, N = (int)pr.dstate,
              G = (int)pr.ngroups;
    launch_begin(adjoint ? "bwd_chunk_adjoint" : "bwd_chunk_state", st);
    using bf = __nv_bfloat16;
    if (pr.dtype == SSD_F32) {
        if (adjoint)
            chunk_state_kernel<float, true><<<grid, kThreads, 0, st>>>(
                (const float *)x, (const float *)dt, A, (const float *)B, S, decay, L, H, P, N, G,
                pr.chunk, nc, pa);
        else
            chunk_state_kernel<float, false><<<grid, kThreads, 0, st>>>(
                (const float *)x, (const float *)dt, A, (const float *)B, S, decay, L, H, P, N, G,
                pr.chunk, nc, pa);
    } else {
        if (adjoint)
            chunk_state_kernel<bf, true><<<grid, kThreads, 0, st>>>(
                (const bf *)x, (const bf *)dt, A, (const bf *)B, S, decay, L, H, P, N, G, pr.chunk,
                nc, pa);
        else
            chunk_state_kernel<bf, false><<<grid, kThreads, 0, st>>>(
                (const bf *)x, (const bf *)dt, A, (const bf *)B, S, decay, L, H, P, N, G, pr.chunk,
                nc, pa);
    }
    launch_end(st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "chunk_state launch");
    return SSD_OK;
}

ssd_status state_chain_launch(const float *S, const float *decays, const float *h0, float *h_in,
                              float *h_total, int64_t batch, int64_t nheads, int PN4, int nparts,
                              int part, cudaStream_t st) {
    dim3 grid((unsigned)((PN4 + kThreads - 1) / kThreads), (unsigned)nheads, (unsigned)batch);
    launch_begin("state_chain", st);
    state_chain_kernel<<<grid, kThreads, 0, st>>>(S, decays, h0, h_in, h_total, batch * nheads,
                                                  PN4, nparts, part);
    launch_end(st);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "state_chain launch");
    return SSD_OK;
}

ssd_status simt_forward(const Problem &pr, const void *x, const void *dt, const float *A,
                        const void *B, const void *C, const float *D, const float *h0,
                        void *y, float *h_final, void *ws, cudaStream_t st, const DtPre &pre) {
    const DtPreArgs pa{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    if (pr.dtype == SSD_F32)
        return forward_t<float>(pr, (const float *)x, (const float *)dt, A, (const float *)B,
                                (const float *)C, D, h0, (float *)y, h_final, ws, st, pa);
    using bf = __nv_bfloat16;
    return forward_t<bf>(pr, (const bf *)x, (const bf *)dt, A, (const bf *)B, (const bf *)C, D,
                         h0, (bf *)y, h_final, ws, st, pa);
}

}  // namespace ssd
