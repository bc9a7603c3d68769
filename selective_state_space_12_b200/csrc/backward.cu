// Backward pass of the layer (the plain forward: decay exp(dt A_h), input
// weight dt), on CUDA cores, by the chunked decomposition of the forward
// ("Mamba-2 — 注意力的远亲", section "两条路各走一半"; "Mamba-2 模型解读",
// section 6.2), with the chunk states recomputed rather than stored
// ("精读笔记 #12：Mamba", section 3.3). For the loss sum dy . y +
// sum dh_final . h_final, per (batch, head) lane and chunk of Q tokens with
// local cumulative log-decay cum_i (total = cum at the last token):
//
//   1. the forward's chunk states and decays; the state pass leaves the
//      state H_c entering each chunk (h0 before the first);
//   2. each chunk's contribution G_c = sum_i exp(cum_i) dy_i (x) C_i to the
//      gradient of its entering state;
//   3. a reverse state pass: R_c = gradient at the END of chunk c
//      (dh_final after the last), R_{c-1} = exp(total_c) R_c + G_c, dh0 the
//      last of these;
//   4. per chunk, with W_ij = exp(cum_i - cum_j) (j <= i), K = C B^T,
//      Z = dy x^T, M = W o dt_j o K, V = W o dt_j o Z, u_j = exp(total -
//      cum_j) dt_j:
//        dx_j = D dy_j + sum_i M_ij dy_i + u_j (R_c B_j)
//        dB_j = sum_i V_ij C_i + u_j (R_c^T x_j)      (per head, summed per group)
//        dC_i = sum_j V_ij B_j + exp(cum_i) (dy_i^T H_c)
//        ddt_j = sum_i W_ij K_ij Z_ij + exp(total - cum_j) x_j^T R_c B_j
//                + A sum_{i >= j} dcum_i
//        dcum_i = sum_j M_ij Z_ij - sum_k M_ki Z_ki + exp(cum_i) dy_i . (C_i H_c^T)
//                 - u_i x_i^T R_c B_i  (+ exp(total) <R_c, H_c> + sum_j u_j x_j^T R_c B_j
//                 at the chunk's last token, through total)
//        dA += sum_j dt_j sum_{i >= j} dcum_i;  dD += sum dy o x
//
// All gradients are fp32. Each chunk's tiles live in shared memory.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace ssd {
namespace {

constexpr int kBT = 256;  // threads per block

// Shared-memory layout of one chunk (floats); rows that vary across lanes
// get one padding column (no bank conflicts on the column walk).
struct BwdSmem {
    int ldX, ldB, ldPN;  // row strides of X, B, and of H / R (N + 1)
    int X, dY, B, C, H, R, M, V, vec, total;
};
__host__ __device__ inline BwdSmem bwd_smem(int Q, int P, int N) {
    BwdSmem s;
    s.ldX = P + 1;
    s.ldB = N + 1;
    s.ldPN = N + 1;
    s.X = 0;
    s.dY = s.X + Q * s.ldX;
    s.B = s.dY + Q * P;
    s.C = s.B + Q * s.ldB;
    s.H = s.C + Q * N;
    s.R = s.H + P * s.ldPN;
    s.M = s.R + P * s.ldPN;
    s.V = s.M + Q * Q;
    s.vec = s.V + Q * Q;        // 10 vectors of Q, then 64 scalars
    s.total = s.vec + 10 * Q + 64;
    return s;
}

// dst (rows x cols, row stride ld) <- lane rows of a (rows_total x cols) tensor
template <typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, int64_t row_stride,
                                          int rows, int valid, int cols) {
    for (int i = threadIdx.x; i < rows * cols; i += blockDim.x) {
        const int r = i / cols, c = i - r * cols;
        dst[r * ld + c] = r < valid ? to_f(src[(int64_t)r * row_stride + c]) : 0.f;
    }
}

__device__ __forceinline__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x < 32) {
        t = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        t = warp_sum(t);
    }
    __syncthreads();
    if (threadIdx.x == 0) red[0] = t;
    __syncthreads();
    const float r = red[0];
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(kBT)
bwd_chunk_kernel(const T *__restrict__ x, const T *__restrict__ dt, const float *__restrict__ A,
                 const T *__restrict__ B, const T *__restrict__ C, const float *__restrict__ D,
                 const float *__restrict__ Hst, const float *__restrict__ Rst,
                 const T *__restrict__ dy, float *__restrict__ dx, float *__restrict__ ddt,
                 float *__restrict__ dBh, float *__restrict__ dCh, float *__restrict__ dA_part,
                 float *__restrict__ dD_part, int L, int H, int P, int N, int G, int Q, int nc) {
    extern __shared__ float sm[];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (H / G);
    const int t0 = c * Q, n = min(Q, L - t0);
    const int tid = threadIdx.x;
    const BwdSmem lay = bwd_smem(Q, P, N);
    float *sX = sm + lay.X, *sdY = sm + lay.dY, *sB = sm + lay.B, *sC = sm + lay.C;
    float *sH = sm + lay.H, *sR = sm + lay.R, *sM = sm + lay.M, *sV = sm + lay.V;
    float *scum = sm + lay.vec, *sdt = scum + Q, *su = sdt + Q, *secum = su + Q;
    float *srow = secum + Q, *scol = srow + Q, *sddir = scol + Q, *sxE = sddir + Q;
    float *syCH = sxE + Q, *sSdt = syCH + Q, *sred = sSdt + Q;  // sred: 64 scalars
    const int64_t lane = (int64_t)b * H + h;
    const int64_t row0 = (int64_t)b * L + t0;
    const int64_t PN = (int64_t)P * N;
    const float Ah = A[h], Dh = D ? D[h] : 0.f;

    // tiles of the chunk (rows past the end of the sequence are zero)
    load_rows(sX, lay.ldX, x + (row0 * H + h) * P, (int64_t)H * P, Q, n, P);
    load_rows(sdY, P, dy + (row0 * H + h) * P, (int64_t)H * P, Q, n, P);
    load_rows(sB, lay.ldB, B + (row0 * G + g) * N, (int64_t)G * N, Q, n, N);
    load_rows(sC, N, C + (row0 * G + g) * N, (int64_t)G * N, Q, n, N);
    load_rows(sH, lay.ldPN, Hst + (lane * nc + c) * PN, (int64_t)N, P, P, N);
    load_rows(sR, lay.ldPN, Rst + (lane * nc + c) * PN, (int64_t)N, P, P, N);
    for (int i = tid; i < Q; i += blockDim.x) {
        sdt[i] = i < n ? to_f(dt[(row0 + i) * H + h]) : 0.f;
        srow[i] = scol[i] = sddir[i] = sxE[i] = syCH[i] = 0.f;
    }
    __syncthreads();
    if (tid == 0) {  // cumulative decay and step (at most Q tokens)
        float cum = 0.f, sd = 0.f;
        for (int i = 0; i < Q; ++i) {
            if (i < n) {
                cum += sdt[i] * Ah;
                sd += sdt[i];
            }
            scum[i] = cum;
            sSdt[i] = sd;
        }
        const float total = n > 0 ? scum[n - 1] : 0.f;
        for (int i = 0; i < Q; ++i) {
            su[i] = i < n ? expf(total - scum[i]) * sdt[i] : 0.f;
            secum[i] = i < n ? expf(scum[i]) : 0.f;
        }
        sred[40] = total;
    }
    __syncthreads();
    const float total = sred[40];

    // M, V and the row / column sums of M o Z, the direct dt term sum_i W K Z.
    // 16 x 16 threads, each a register tile of rows ti + 16 a and columns
    // tj + 16 b (a, b < Q / 16) of K = C B^T and Z = dy x^T
    const int RQ = Q / 16;  // 1, 2 or 4
    {
        const int ti = tid >> 4, tj = tid & 15;
        float Kt[4][4], Zt[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) Kt[a][bb] = Zt[a][bb] = 0.f;
        for (int k = 0; k < N; ++k) {
            float cv[4], bv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                cv[a] = a < RQ ? sC[(ti + 16 * a) * N + k] : 0.f;
                bv[a] = a < RQ ? sB[(tj + 16 * a) * lay.ldB + k] : 0.f;
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) Kt[a][bb] = fmaf(cv[a], bv[bb], Kt[a][bb]);
        }
        for (int k = 0; k < P; ++k) {
            float yv[4], xv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                yv[a] = a < RQ ? sdY[(ti + 16 * a) * P + k] : 0.f;
                xv[a] = a < RQ ? sX[(tj + 16 * a) * lay.ldX + k] : 0.f;
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) Zt[a][bb] = fmaf(yv[a], xv[bb], Zt[a][bb]);
        }
        float rows[4] = {0.f, 0.f, 0.f, 0.f}, cols[4] = {0.f, 0.f, 0.f, 0.f};
        float ddir[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int a = 0; a < 4; ++a) {
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                if (a >= RQ || bb >= RQ) continue;
                const int i = ti + 16 * a, j = tj + 16 * bb;
                float Mv = 0.f, Vv = 0.f;
                if (j <= i && i < n) {
                    const float W = expf(scum[i] - scum[j]);
                    Mv = W * sdt[j] * Kt[a][bb];
                    Vv = W * sdt[j] * Zt[a][bb];
                    const float mz = Mv * Zt[a][bb];
                    rows[a] += mz;
                    cols[bb] += mz;
                    ddir[bb] = fmaf(W * Kt[a][bb], Zt[a][bb], ddir[bb]);
                }
                sM[i * Q + j] = Mv;
                sV[i * Q + j] = Vv;
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            if (a >= RQ) continue;
            atomicAdd(&srow[ti + 16 * a], rows[a]);
            atomicAdd(&scol[tj + 16 * a], cols[a]);
            atomicAdd(&sddir[tj + 16 * a], ddir[a]);
        }
    }
    __syncthreads();

    // dx_j = D dy_j + sum_i M_ij dy_i + u_j (R B_j), with x_j . (R B_j) summed
    // into sxE, and dy_j . (C_j H^T) summed into syCH: register tiles of rows
    // tj + 16 a (a < Q / 16) and columns tp + 16 bb (bb < P / 16 <= 8)
    {
        const int tj = tid >> 4, tp = tid & 15;
        const int RP = P / 16;
        float m[4][8], e[4][8], ch[4][8];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) m[a][bb] = e[a][bb] = ch[a][bb] = 0.f;
        for (int i = 0; i < n; ++i) {
            float ma[4], yb[8];
#pragma unroll
            for (int a = 0; a < 4; ++a) ma[a] = a < RQ ? sM[i * Q + tj + 16 * a] : 0.f;
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) yb[bb] = bb < RP ? sdY[i * P + tp + 16 * bb] : 0.f;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) m[a][bb] = fmaf(ma[a], yb[bb], m[a][bb]);
        }
        for (int k = 0; k < N; ++k) {
            float ba[4], ca[4], rb[8], hb[8];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = tj + 16 * a;
                ba[a] = a < RQ ? sB[r * lay.ldB + k] : 0.f;
                ca[a] = a < RQ ? sC[r * N + k] : 0.f;
            }
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                const int p = tp + 16 * bb;
                rb[bb] = bb < RP ? sR[p * lay.ldPN + k] : 0.f;
                hb[bb] = bb < RP ? sH[p * lay.ldPN + k] : 0.f;
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) {
                    e[a][bb] = fmaf(ba[a], rb[bb], e[a][bb]);
                    ch[a][bb] = fmaf(ca[a], hb[bb], ch[a][bb]);
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int j = tj + 16 * a;
            if (a >= RQ || j >= n) continue;
            float xe = 0.f, ych = 0.f;
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                if (bb >= RP) continue;
                const int p = tp + 16 * bb;
                dx[(row0 + j) * H * (int64_t)P + (int64_t)h * P + p] =
                    fmaf(Dh, sdY[j * P + p], m[a][bb]) + su[j] * e[a][bb];
                xe = fmaf(sX[j * lay.ldX + p], e[a][bb], xe);
                ych = fmaf(sdY[j * P + p], ch[a][bb], ych);
            }
            atomicAdd(&sxE[j], xe);
            atomicAdd(&syCH[j], ych);
        }
    }
    // per-head dB_j = sum_i V_ij C_i + u_j (R^T x_j); dC_i = sum_j V_ij B_j + e^cum_i (dy_i^T H):
    // register tiles of rows tr + 16 a (a < Q / 16) and columns kb + tk + 16 c
    // (c < 8), 128 columns per pass; V is zero outside its triangle, so the
    // token loops run over the whole chunk
    {
        const int tr = tid >> 4, tk = tid & 15;
        for (int kb = 0; kb < N; kb += 128) {
            float v[4][8], v2[4][8];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) v[a][cc] = v2[a][cc] = 0.f;
            for (int t = 0; t < n; ++t) {
                float va[4], vb[4], ck[8], bk[8];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = tr + 16 * a;
                    va[a] = a < RQ ? sV[t * Q + r] : 0.f;  // V[t][r]
                    vb[a] = a < RQ ? sV[r * Q + t] : 0.f;  // V[r][t]
                }
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int k = kb + tk + 16 * cc;
                    ck[cc] = k < N ? sC[t * N + k] : 0.f;
                    bk[cc] = k < N ? sB[t * lay.ldB + k] : 0.f;
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        v[a][cc] = fmaf(va[a], ck[cc], v[a][cc]);
                        v2[a][cc] = fmaf(vb[a], bk[cc], v2[a][cc]);
                    }
            }
            float f[4][8], yh[4][8];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) f[a][cc] = yh[a][cc] = 0.f;
            for (int p = 0; p < P; ++p) {
                float xa[4], ya[4], rk[8], hk[8];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = tr + 16 * a;
                    xa[a] = a < RQ ? sX[r * lay.ldX + p] : 0.f;
                    ya[a] = a < RQ ? sdY[r * P + p] : 0.f;
                }
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int k = kb + tk + 16 * cc;
                    rk[cc] = k < N ? sR[p * lay.ldPN + k] : 0.f;
                    hk[cc] = k < N ? sH[p * lay.ldPN + k] : 0.f;
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        f[a][cc] = fmaf(xa[a], rk[cc], f[a][cc]);
                        yh[a][cc] = fmaf(ya[a], hk[cc], yh[a][cc]);
                    }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = tr + 16 * a;
                if (a >= RQ || r >= n) continue;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int k = kb + tk + 16 * cc;
                    if (k >= N) continue;
                    const int64_t o = ((row0 + r) * H + h) * (int64_t)N + k;
                    dBh[o] = v[a][cc] + su[r] * f[a][cc];
                    dCh[o] = v2[a][cc] + secum[r] * yh[a][cc];
                }
            }
        }
    }
    // <R, H> and sum dy o x
    float rh = 0.f, yx = 0.f;
    for (int idx = tid; idx < P * N; idx += blockDim.x) {
        const int p = idx / N, k = idx - p * N;
        rh = fmaf(sR[p * lay.ldPN + k], sH[p * lay.ldPN + k], rh);
    }
    for (int idx = tid; idx < n * P; idx += blockDim.x) {
        const int i = idx / P, p = idx - i * P;
        yx = fmaf(sdY[i * P + p], sX[i * lay.ldX + p], yx);
    }
    rh = block_sum(rh, sred);
    yx = block_sum(yx, sred);
    __syncthreads();
    if (tid == 0) {
        float dtot = expf(total) * rh;
        for (int j = 0; j < n; ++j) dtot = fmaf(su[j], sxE[j], dtot);
        float sdc = 0.f, dAp = 0.f;
        for (int i = n - 1; i >= 0; --i) {
            float dc = srow[i] - scol[i] + secum[i] * syCH[i] - su[i] * sxE[i];
            if (i == n - 1) dc += dtot;
            sdc += dc;
            ddt[(row0 + i) * H + h] = sddir[i] + expf(total - scum[i]) * sxE[i] + Ah * sdc;
            dAp = fmaf(sdt[i], sdc, dAp);
        }
        dA_part[lane * nc + c] = dAp;
        dD_part[lane * nc + c] = yx;
    }
}

// R (lanes, nc, P*N): each chunk's G on entry, the gradient at the chunk's
// end on exit; dh0 receives the gradient at the start of the first chunk.
__global__ void __launch_bounds__(kBT)
reverse_pass_kernel(float *__restrict__ R, const float *__restrict__ decay,
                    const float *dh_final, float *dh0, int H, int PN4, int nc) {
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (q >= PN4) return;
    const int64_t lane = (int64_t)b * H + h;
    float4 st = make_float4(0.f, 0.f, 0.f, 0.f);
    if (dh_final) st = reinterpret_cast<const float4 *>(dh_final + lane * PN4 * 4)[q];
    float4 *Rp = reinterpret_cast<float4 *>(R + lane * nc * (int64_t)PN4 * 4);
    const float *dp = decay + lane * nc;
    // the next (earlier) chunk's load goes out before this chunk's update
    float4 g_next = make_float4(0.f, 0.f, 0.f, 0.f);
    float d_next = 0.f;
    if (nc > 0) {
        g_next = Rp[(int64_t)(nc - 1) * PN4 + q];
        d_next = dp[nc - 1];
    }
    for (int c = nc - 1; c >= 0; --c) {
        const float4 gc = g_next;
        const float d = d_next;
        if (c > 0) {
            g_next = Rp[(int64_t)(c - 1) * PN4 + q];
            d_next = dp[c - 1];
        }
        Rp[(int64_t)c * PN4 + q] = st;
        st.x = fmaf(d, st.x, gc.x);
        st.y = fmaf(d, st.y, gc.y);
        st.z = fmaf(d, st.z, gc.z);
        st.w = fmaf(d, st.w, gc.w);
    }
    if (dh0) reinterpret_cast<float4 *>(dh0 + lane * PN4 * 4)[q] = st;
}

// out[b][t][g][n] = sum over the heads of group g of per_head[b][t][h][n]
__global__ void __launch_bounds__(kBT)
group_sum_kernel(const float *__restrict__ per_head, float *__restrict__ out, int64_t rows,
                 int H, int G, int N) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = rows * G * N;
    if (i >= total) return;
    const int64_t row = i / ((int64_t)G * N);
    const int rem = (int)(i - row * G * N), g = rem / N, k = rem - g * N;
    const int hpg = H / G;
    float s = 0.f;
    for (int hh = 0; hh < hpg; ++hh) s += per_head[(row * H + g * hpg + hh) * (int64_t)N + k];
    out[i] = s;
}

// out[h] = sum over batch and chunks of part[(b H + h) nc + c]
__global__ void __launch_bounds__(kBT)
head_sum_kernel(const float *__restrict__ part, float *__restrict__ out, int batch, int H,
                int nc) {
    __shared__ float red[64];
    const int h = blockIdx.x;
    float s = 0.f;
    for (int i = threadIdx.x; i < batch * nc; i += blockDim.x) {
        const int b = i / nc, c = i - b * nc;
        s += part[((int64_t)b * H + h) * nc + c];
    }
    s = block_sum(s, red);
    if (threadIdx.x == 0) out[h] = s;
}

struct BwdWs {
    float *Hst, *decay, *R, *decay2, *dBh, *dCh, *dA_part, *dD_part;
    size_t bytes;
};

// per_head: room for the per-head dB and dC that the CUDA-core path sums over
// each group afterwards (the tensor-core path adds into dB and dC directly).
BwdWs bwd_ws(const Problem &pr, int Q, void *base, bool per_head_sums) {
    const size_t lanes = (size_t)(pr.batch * pr.nheads);
    const size_t nc = (size_t)((pr.seqlen + Q - 1) / Q);
    const size_t PN = (size_t)(pr.headdim * pr.dstate);
    const size_t per_head =
        per_head_sums ? (size_t)(pr.batch * pr.seqlen * pr.nheads * pr.dstate) : 0;
    size_t off = 0;
    char *p = static_cast<char *>(base);
    auto take = [&](size_t floats) {
        float *r = reinterpret_cast<float *>(p ? p + off : nullptr);
        off += align256(floats * 4);
        return r;
    };
    BwdWs w;
    w.Hst = take(lanes * nc * PN);
    w.decay = take(lanes * nc);
    w.R = take(lanes * nc * PN);
    w.decay2 = take(lanes * nc);
    w.dBh = take(per_head);
    w.dCh = take(per_head);
    w.dA_part = take(lanes * nc);
    w.dD_part = take(lanes * nc);
    w.bytes = off;
    return w;
}

size_t smem_floats(int Q, int P, int N) { return (size_t)bwd_smem(Q, P, N).total; }

}  // namespace

// The tensor-core path unless LIBSSD_BACKWARD_PATH=simt; =tc requires it.
static bool use_tc_backward(const Problem &pr) {
    const char *e = getenv("LIBSSD_BACKWARD_PATH");
    if (e && strcmp(e, "simt") == 0) return false;
    return tc_backward_supported(pr);
}

// The tensor-core chunk states as lane-walking chains where the problem has
// the lanes for them; LIBSSD_BACKWARD_CHAIN=0 or 1 overrides the choice
// (tests and profiling).
static bool use_tc_chain(const Problem &pr) {
    const char *e = getenv("LIBSSD_BACKWARD_CHAIN");
    if (e && strcmp(e, "0") == 0) return false;
    if (e && strcmp(e, "1") == 0) return true;
    return tc_chain_pays(pr);
}

int backward_chunk(const Problem &pr) {
    if (use_tc_backward(pr)) return 128;
    for (int Q : {64, 32, 16}) {
        if (smem_floats(Q, (int)pr.headdim, (int)pr.dstate) * 4 <= 227 * 1024) return Q;
    }
    return 0;
}

size_t backward_workspace_bytes(const Problem &pr) {
    const int Q = backward_chunk(pr);
    if (Q == 0) return 0;
    return bwd_ws(pr, Q, nullptr, !use_tc_backward(pr)).bytes;
}

ssd_status backward_launch(const Problem &pr_in, const void *x, const void *dt, const float *A,
                           const void *B, const void *C, const float *D, const float *h0,
                           const void *dy, const float *dh_final, float *dx, float *ddt,
                           float *dA, float *dB, float *dC, float *dD, float *dh0, void *ws,
                           cudaStream_t st) {
    const int Q = backward_chunk(pr_in);
    if (Q == 0) return fail(SSD_ERR_UNSUPPORTED, "backward: headdim x dstate too large");
    Problem pr = pr_in;
    pr.chunk = Q;
    const int nc = (int)pr.nchunks();
    const int H = (int)pr.nheads, P = (int)pr.headdim, N = (int)pr.dstate, G = (int)pr.ngroups;
    const int PN4 = P * N / 4;
    const bool tc = use_tc_backward(pr_in);
    const BwdWs w = bwd_ws(pr, Q, ws, !tc);
    ssd_status s;
    cudaError_t e;
    if (tc && use_tc_chain(pr)) {
        // 1-3 on the tensor cores, each chain in one pass along the lanes: the
        // state entering each chunk, then the gradient at each chunk's end and dh0
        if ((s = tc_state_chain(pr, x, dt, A, B, h0, w.Hst, nullptr, false, st)) != SSD_OK)
            return s;
        if ((s = tc_state_chain(pr, dy, dt, A, C, dh_final, w.R, dh0, true, st)) != SSD_OK)
            return s;
    } else {
        // 1. forward chunk states -> the state entering each chunk
        if ((s = tc ? tc_chunk_states(pr, x, dt, A, B, w.Hst, w.decay, false, st)
                    : chunk_states_launch(pr, x, dt, A, B, w.Hst, w.decay, false, st)) != SSD_OK)
            return s;
        if ((s = state_pass_launch(w.Hst, w.decay, h0, nullptr, pr.batch, pr.nheads, PN4, nc,
                                   st)) != SSD_OK)
            return s;
        // 2. each chunk's contribution to its entering state's gradient
        if ((s = tc ? tc_chunk_states(pr, dy, dt, A, C, w.R, w.decay2, true, st)
                    : chunk_states_launch(pr, dy, dt, A, C, w.R, w.decay2, true, st)) != SSD_OK)
            return s;
        // 3. reverse pass: the gradient at each chunk's end, and dh0
        dim3 grid((unsigned)((PN4 + kBT - 1) / kBT), (unsigned)H, (unsigned)pr.batch);
        launch_begin("bwd_reverse_pass", st);
        if (nc > 0 || dh0)
            reverse_pass_kernel<<<grid, kBT, 0, st>>>(w.R, w.decay, dh_final, dh0, H, PN4, nc);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "reverse pass launch");
    }
    // 4. per-chunk gradients
    {
        const char *e2 = getenv("LIBSSD_BACKWARD_PATH");
        if (e2 && strcmp(e2, "tc") == 0 && !tc)
            return fail(SSD_ERR_UNSUPPORTED, "backward: the tensor-core path does not take these sizes");
    }
    if (nc > 0 && tc) {
        // every head adds its share of dB and dC
        const size_t gbytes = (size_t)(pr.batch * pr.seqlen * G * N) * 4;
        if ((e = cudaMemsetAsync(dB, 0, gbytes, st)) != cudaSuccess ||
            (e = cudaMemsetAsync(dC, 0, gbytes, st)) != cudaSuccess)
            return cuda_fail(e, "zeroing dB and dC");
        if ((s = tc_backward_chunks(pr, x, dt, A, B, C, D, dy, w.Hst, w.R, dx, ddt, dB, dC,
                                    w.dA_part, w.dD_part, st)) != SSD_OK)
            return s;
    } else if (nc > 0) {
        const size_t smem = smem_floats(Q, P, N) * 4;
        dim3 grid((unsigned)nc, (unsigned)H, (unsigned)pr.batch);
        launch_begin("bwd_chunk", st);
        if (pr.dtype == SSD_F32) {
            if ((e = cudaFuncSetAttribute(bwd_chunk_kernel<float>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem)) != cudaSuccess)
                return cuda_fail(e, "bwd_chunk smem");
            bwd_chunk_kernel<float><<<grid, kBT, smem, st>>>(
                (const float *)x, (const float *)dt, A, (const float *)B, (const float *)C, D,
                w.Hst, w.R, (const float *)dy, dx, ddt, w.dBh, w.dCh, w.dA_part, w.dD_part,
                (int)pr.seqlen, H, P, N, G, Q, nc);
        } else {
            using bf = __nv_bfloat16;
            if ((e = cudaFuncSetAttribute(bwd_chunk_kernel<bf>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem)) != cudaSuccess)
                return cuda_fail(e, "bwd_chunk smem");
            bwd_chunk_kernel<bf><<<grid, kBT, smem, st>>>(
                (const bf *)x, (const bf *)dt, A, (const bf *)B, (const bf *)C, D, w.Hst, w.R,
                (const bf *)dy, dx, ddt, w.dBh, w.dCh, w.dA_part, w.dD_part, (int)pr.seqlen, H, P,
                N, G, Q, nc);
        }
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd_chunk launch");
    }
    // 5. sums over the heads of a group and over batch and chunks
    const int64_t rows = pr.batch * pr.seqlen;
    const int64_t gsz = rows * G * N;
    launch_begin("bwd_reduce", st);
    if (gsz > 0 && !tc) {  // the tensor-core path added into dB and dC already
        const unsigned nb = (unsigned)((gsz + kBT - 1) / kBT);
        if (dB) group_sum_kernel<<<nb, kBT, 0, st>>>(w.dBh, dB, rows, H, G, N);
        if (dC) group_sum_kernel<<<nb, kBT, 0, st>>>(w.dCh, dC, rows, H, G, N);
    }
    if (nc > 0) {
        if (dA) head_sum_kernel<<<H, kBT, 0, st>>>(w.dA_part, dA, (int)pr.batch, H, nc);
        if (dD) head_sum_kernel<<<H, kBT, 0, st>>>(w.dD_part, dD, (int)pr.batch, H, nc);
    } else {
        if (dA && (e = cudaMemsetAsync(dA, 0, (size_t)H * 4, st)) != cudaSuccess)
            return cuda_fail(e, "dA");
        if (dD && (e = cudaMemsetAsync(dD, 0, (size_t)H * 4, st)) != cudaSuccess)
            return cuda_fail(e, "dD");
    }
    launch_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd reduce launch");
    return SSD_OK;
}

}  // namespace ssd
