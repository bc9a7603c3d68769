// Tensor-core backward of the plain layer for bf16 I/O, P = 64, N = 128,
// 128-token chunks ("精读笔记 #12：Mamba" section 3.3: the chunk states are
// recomputed, not stored). Two kernels: the chain of chunk states along each
// lane (the state entering each chunk, or the gradient at each chunk's end),
// and the per-chunk gradients. The second runs one persistent CTA of eight
// warps per SM over the (chunk, head, batch) items; thread 0 issues the TMA
// loads and MMAs. Token t of the chunk is TMEM lane t, which warps t / 32 and
// t / 32 + 4 can both reach: the row's two threads (halves 0 and 1) split its
// column groups and head-dim columns.
//
// Per chunk (cum in log2 units, c_t; tot = c at the chunk's last token; R the
// gradient at the chunk's end and H the state entering it, both P x N):
//   K^T = B C^T, Z^T = X dY^T, Z = dY X^T,  B R^T,  C H^T
//   M^T_{t,i} = 2^(c_i - c_t) dt_t K_{i,t}   (i >= t)
//   V_ij      = 2^(c_i - c_j) dt_j Z_ij      (j <= i), and its transpose
//   dX = M^T dY
// and per token t, with e_t = 2^c_t, u_t = 2^(tot - c_t) dt_t:
//   a_t    = sum_i W_it K_it Z_it                  (row of the transposed view)
//   s_t    = sum_j M_tj Z_tj                        (cross-thread: warp transpose-sum)
//   dcum_t = s_t - dt_t a_t + e_t dY_t.CH_t - u_t X_t.BR_t
//            (+ 2^tot <R, H> + sum_j u_j X_j.BR_j at the last token)
//   ddt_t  = a_t + 2^(tot - c_t) X_t.BR_t + A sum_{k >= t} dcum_k
//   dx_t   = D dY_t + dX_t + u_t BR_t
//   dB_j   = sum_i V_ij C_i + u_j (X R)_j      dC_i = sum_j V_ij B_j + e_i (dY H)_i
// Each head adds its share of dB and dC into the group's (fp32 reductions in
// L2; the order of the heads' additions is not fixed).
#include <cudaTypedefs.h>
#include <stddef.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr int kThreads = 128;      // chain kernel: one thread per state row
constexpr int kThreads2 = 256;     // per-chunk gradient kernel: two threads per row
constexpr int kTile = 128 * 128;  // 128 rows x 128 bytes
constexpr long long kWait = 4000000000LL;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kErrBwdLoad = 0x201, kErrBwdMma = 0x202;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Lane l returns the warp's sum of v[l] (v[k] is this lane's value for index k).
__device__ __forceinline__ float transpose_sum32(float (&v)[32]) {
    const int l = threadIdx.x & 31;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool up = (l & off) != 0;
#pragma unroll
        for (int k = 0; k < off; ++k) {
            const float send = up ? v[k] : v[k + off];
            const float keep = up ? v[k + off] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

// Sum over all threads of a 256-thread block, through red (8 floats that no
// thread reads or writes around the call: one barrier).
__device__ __forceinline__ float block_sum256(float v, float *red) {
    v = warp_sum(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += red[k];
    return s;
}

// The block's sums of the four values in s, and the inclusive scan of v over
// the 128 rows of each half of the block (as row_scan256), in one exchange
// through buf (5 x 8 floats that no thread reads or writes around the call:
// one barrier).
__device__ __forceinline__ float4 block_sums_row_scan256(float4 s, float v, float &scan,
                                                         float (*buf)[8]) {
    const int l = threadIdx.x & 31, w = threadIdx.x >> 5;
    s.x = warp_sum(s.x);
    s.y = warp_sum(s.y);
    s.z = warp_sum(s.z);
    s.w = warp_sum(s.w);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, v, off);
        if (l >= off) v += o;
    }
    if (l == 0) {
        buf[0][w] = s.x;
        buf[1][w] = s.y;
        buf[2][w] = s.z;
        buf[3][w] = s.w;
    }
    if (l == 31) buf[4][w] = v;
    __syncthreads();
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        r.x += buf[0][k];
        r.y += buf[1][k];
        r.z += buf[2][k];
        r.w += buf[3][k];
    }
    float base = 0.f;
    for (int k = w & ~3; k < w; ++k) base += buf[4][k];
    scan = v + base;
    return r;
}

// Inclusive scan over the 128 rows in a 256-thread block: each half of the
// block (threads 0-127, 128-255) scans its own values by row.
__device__ __forceinline__ float row_scan256(float v, float *tmp) {
    const int l = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, v, off);
        if (l >= off) v += o;
    }
    __syncthreads();
    if (l == 31) tmp[w] = v;
    __syncthreads();
    float base = 0.f;
    for (int k = w & ~3; k < w; ++k) base += tmp[k];
    return v + base;
}

// inclusive scan over the 128 threads (t = threadIdx.x)
__device__ __forceinline__ float block_scan128(float v, float *tmp) {
    const int l = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, v, off);
        if (l >= off) v += o;
    }
    __syncthreads();
    if (l == 31) tmp[w] = v;
    __syncthreads();
    float base = 0.f;
    for (int k = 0; k < w; ++k) base += tmp[k];
    return v + base;
}

// bounded wait (`limit` clock cycles, the library's wait bound); on time-out
// sets the abort flag and an error code. The phase is tested without blocking
// and the bound checked before each hardware-suspended try: a try can sleep
// until the phase completes, so a bound shorter than the wait would otherwise
// never be seen.
__device__ __noinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, int *abort,
                                          unsigned int *err, long long limit, unsigned code) {
    const long long t0 = clock64();
    while (true) {
        if (mbar_test_wait(bar, parity)) return true;
        if (*(volatile int *)abort) return false;
        if (clock64() - t0 > limit) {
            *(volatile int *)abort = 1;
            atomicOr(err, code);
            return false;
        }
        if (mbar_try_wait(bar, parity)) return true;
    }
}

constexpr int kHalfTile = 64 * 128;  // 64 rows x 128 bytes

// 16-byte chunk cc (0..15) of row p of a P x N fp32 matrix (columns 8 cc ..
// 8 cc + 7, given as v0, v1) into the two-atom bf16 hi + lo layout.
__device__ __forceinline__ void put_pn_row_chunk(unsigned char *hi, unsigned char *lo, float4 v0,
                                                 float4 v1, int p, int cc) {
    const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        split_bf16x2(f[2 * k], f[2 * k + 1], wh[k], wl[k]);
    }
    const int atom = cc >> 3, ch = cc & 7;
    const uint32_t off = (uint32_t)atom * kHalfTile + swz(p, ch);
    *reinterpret_cast<uint4 *>(hi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
}

// ---------------------------------------------------------------------------
// The per-chunk gradients: dx, ddt, the chunk's parts of dA and dD, and the
// head's share of dB and dC, from one load of the chunk's tiles (one kernel
// instead of a dx kernel and a dB/dC kernel that loaded the same tiles: 747 +
// 859 -> 1243 us on the 2.7B-style layer). One CTA of 256 threads (two per
// token row) per SM walks the (chunk, head, batch) items, each item's fp32
// states requested one item ahead (1243 -> 1190 us).
// TMEM, in order of use:
//   0-127    K^T = B C^T -> M^T (hi + lo), then the dB accumulator V^T C
//   128-255  Z^T = X dY^T -> V^T (hi + lo), then the dC accumulator V B
//   256-383  Z = dY X^T -> V (hi + lo)
//   384-447  B R^T; 448-511 C H^T, then dX = M^T dY
//   384-511  X R (after dx is out), then dY H
// R and H are P rows x N (two 64-column atoms, bf16 hi + lo): an MN-major B
// operand for X R and dY H, a K-major one for B R^T and C H^T. Shared memory:
// the six input tiles (160 KB) and a 32 KB dx staging tile; dB is staged
// where C and R were, dC where X, dY and B were.
constexpr int oMX = 0, oMdY = kTile, oMB = 2 * kTile, oMC = 4 * kTile;
constexpr int oMRh = 6 * kTile, oMRl = oMRh + 2 * kHalfTile;
constexpr int oMHh = oMRl + 2 * kHalfTile, oMHl = oMHh + 2 * kHalfTile;
constexpr int oMDX = oMHl + 2 * kHalfTile;  // 160 KB
constexpr int oMSmall = oMDX + 2 * kTile;   // 192 KB

struct SmallM {
    float c2[kQ];
    float dt[kQ];
    float colT[kQ];        // 2^(c_i - c_{32 I}), I = i / 32
    float colV[4][kQ];     // [q][j] = 2^(c_{32 q} - c_j) dt_j, j < 32 q
    float spart[4][kQ];    // per lane quarter: partial sums of M_tj Z_tj over its rows
    float part[3][2][kQ];  // per row and half: sum_i W K Z, X.BR, dY.CH
    float scan[8];
    float red[8];
    float red5[5][8];
    uint64_t full, mma_a, mma_b, mma_c, mma_d;
    uint32_t tmem_base;
    int abort;
};
constexpr int smemM_bytes() { return oMSmall + (int)sizeof(SmallM) + 1024; }
static_assert(smemM_bytes() <= 227 * 1024, "shared memory");

struct BwdMArgs {
    const __nv_bfloat16 *dt;
    const float *A, *D;
    const float *Hst, *Rst;  // per (lane, chunk): state entering / gradient at the end, [p][n]
    float *ddt, *dA_part, *dD_part;
    unsigned int *err;
    long long wait;  // bound of each wait, clock cycles
    int L, H, G, nc, batch;
};

__global__ void __launch_bounds__(kThreads2, 1)
tc_bwd_chunk_grads_kernel(const __grid_constant__ CUtensorMap mX,
                          const __grid_constant__ CUtensorMap mdY,
                          const __grid_constant__ CUtensorMap mB,
                          const __grid_constant__ CUtensorMap mC,
                          const __grid_constant__ CUtensorMap mDX,
                          const __grid_constant__ CUtensorMap mDB,
                          const __grid_constant__ CUtensorMap mDC, const BwdMArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    SmallM *sm = reinterpret_cast<SmallM *>(smem + oMSmall);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = tid & (kQ - 1);   // this thread's row (token)
    const int half = tid >> 7;      // which half of the row's columns
    const int q = warp & 3;         // TMEM lane quarter
    const long long PN = (long long)kP * kN;
    const long long items = (long long)a.nc * a.H * a.batch;

    if (tid == 0) {
        mbar_init(&sm->full, 1);
        mbar_init(&sm->mma_a, 1);
        mbar_init(&sm->mma_b, 1);
        mbar_init(&sm->mma_c, 1);
        mbar_init(&sm->mma_d, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const uint32_t base = smem_u32(smem);
    int *ab = &sm->abort;
    if (tid == 0) tma_prefetch_desc(&mX);

    // The CTA walks items (chunk fastest, then head, then batch) with the
    // grid's stride; item i's end gradient R and entering state H (fp32,
    // P x N, at i * P * N) are loaded into registers during item i - stride,
    // so that their latency hides behind a whole item. 64 rows x 16 chunks per
    // matrix: 4 (row, chunk) items per thread.
    float4 rv[4][2], hv[4][2];
    auto load_states = [&](long long item) {
        const float *R = a.Rst + item * PN;
        const float *Hs = a.Hst + item * PN;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int it = tid + kThreads2 * i;
            const long long o = (long long)(it >> 4) * kN + 8 * (it & 15);
            rv[i][0] = __ldcg(reinterpret_cast<const float4 *>(R + o));
            rv[i][1] = __ldcg(reinterpret_cast<const float4 *>(R + o + 4));
            hv[i][0] = __ldcg(reinterpret_cast<const float4 *>(Hs + o));
            hv[i][1] = __ldcg(reinterpret_cast<const float4 *>(Hs + o + 4));
        }
    };
    long long item = blockIdx.x;
    if (item < items) load_states(item);
#pragma unroll 1
    for (int iter = 0; item < items; ++iter, item += gridDim.x) {
        const uint32_t ph = iter & 1;  // every barrier completes one phase per item
        const int c = (int)(item % a.nc);
        const long long lane_bh = item / a.nc;
        const int h = (int)(lane_bh % a.H), b = (int)(lane_bh / a.H);
        const int g = h / (a.H / a.G);
        const int t0 = c * kQ;
        const int n = min(kQ, a.L - t0);
        const float Ah = a.A[h], Dh = a.D ? a.D[h] : 0.f;
        bool iss_a = false, iss_b = false, iss_c = false, iss_d = false;  // thread 0

        if (tid == 0) {
            mbar_arrive_expect_tx(&sm->full, 6 * kTile);
            tma_load_4d(smem + oMX, &mX, &sm->full, 0, h, t0, b);
            tma_load_4d(smem + oMdY, &mdY, &sm->full, 0, h, t0, b);
            tma_load_4d(smem + oMB, &mB, &sm->full, 0, g, t0, b);
            tma_load_4d(smem + oMB + kTile, &mB, &sm->full, 64, g, t0, b);
            tma_load_4d(smem + oMC, &mC, &sm->full, 0, g, t0, b);
            tma_load_4d(smem + oMC + kTile, &mC, &sm->full, 64, g, t0, b);
        }

        // steps and cumulative log2-decay (tokens past the end: dt = 0), the same
        // scan in both halves
        const float dtt = t < n ? __bfloat162float(a.dt[((long long)b * a.L + t0 + t) * a.H + h]) : 0.f;
        const float c2t = row_scan256(dtt * Ah * kLog2e, sm->scan);
        if (half == 0) {
            sm->c2[t] = c2t;
            sm->dt[t] = dtt;
        }
        // With A <= 0 and no negative step, c falls along the chunk, and the
        // decays of the column groups off the row's own split into a row factor
        // and a column factor, both at most 1, so neither overflows and a factor
        // underflows only where the decay itself is below 2^-126:
        //   M^T, V^T, group J > q:  [2^(c_i - c_{32 J})] * 2^(c_{32 J} - c_t)
        //   V,        group J < q:  2^(c_t - c_{32 q}) * [2^(c_{32 q} - c_j) dt_j]
        const bool mono = __syncthreads_and(dtt >= 0.f) && Ah <= 0.f;
        if (half == 1) {
            sm->colT[t] = fast_exp2(c2t - sm->c2[t & ~31]);
        } else {
#pragma unroll
            for (int qq = 1; qq < 4; ++qq)
                if (t < 32 * qq) sm->colV[qq][t] = fast_exp2(sm->c2[32 * qq] - c2t) * dtt;
        }

        // R and H as P rows x N bf16 hi + lo, and this thread's part of <R, H>;
        // then the next item's states are requested
        float rh_dot = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int it = tid + kThreads2 * i;
#pragma unroll
            for (int u = 0; u < 2; ++u)
                rh_dot += rv[i][u].x * hv[i][u].x + rv[i][u].y * hv[i][u].y +
                          rv[i][u].z * hv[i][u].z + rv[i][u].w * hv[i][u].w;
            put_pn_row_chunk(smem + oMRh, smem + oMRl, rv[i][0], rv[i][1], it >> 4, it & 15);
            put_pn_row_chunk(smem + oMHh, smem + oMHl, hv[i][0], hv[i][1], it >> 4, it & 15);
        }
        if (item + gridDim.x < items) load_states(item + gridDim.x);
        fence_proxy_async_smem();
        __syncthreads();
        const float tot2 = sm->c2[kQ - 1];

        constexpr uint32_t iSq = idesc_bf16(128, 128, false, false);
        constexpr uint32_t iOutK = idesc_bf16(128, 64, false, false);
        constexpr uint32_t iDiag = idesc_bf16(128, 64, false, true);
        constexpr uint32_t iWideMN = idesc_bf16(128, 128, false, true);
        const uint64_t dX = sdesc_sw128(base + oMX, 16, 1024);
        const uint64_t ddY = sdesc_sw128(base + oMdY, 16, 1024);
        if (tid == 0) {
            if (wait_bounded(&sm->full, ph, ab, a.err, a.wait, kErrBwdLoad)) {
                tc_fence_after();
                const uint64_t dB = sdesc_sw128(base + oMB, 16, 1024);
                const uint64_t dC = sdesc_sw128(base + oMC, 16, 1024);
                // K^T = B C^T (K = state dim, two atoms)
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t off = ((k >> 2) * kTile + (k & 3) * 32) >> 4;
                    mma_ss(tmem + 0, dB + off, dC + off, iSq, k > 0);
                }
                // Z^T = X dY^T and Z = dY X^T (K = head dim, one atom)
#pragma unroll
                for (int k = 0; k < kP / 16; ++k)
                    mma_ss(tmem + 128, dX + ((k * 32) >> 4), ddY + ((k * 32) >> 4), iSq, k > 0);
#pragma unroll
                for (int k = 0; k < kP / 16; ++k)
                    mma_ss(tmem + 256, ddY + ((k * 32) >> 4), dX + ((k * 32) >> 4), iSq, k > 0);
                // B R^T and C H^T: the P x N tiles as K-major B operands (K = state
                // dim, two 8 KB atoms), hi then lo into one accumulator
                const uint32_t hl[4] = {base + oMRh, base + oMRl, base + oMHh, base + oMHl};
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint64_t dA_ = (s < 2) ? dB : dC;
                    const uint64_t dS = sdesc_sw128(hl[s], 16, 1024);
                    const uint32_t acc = tmem + (s < 2 ? 384 : 448);
#pragma unroll
                    for (int k = 0; k < kN / 16; ++k) {
                        const uint32_t offa = ((k >> 2) * kTile + (k & 3) * 32) >> 4;
                        const uint32_t offs = ((k >> 2) * kHalfTile + (k & 3) * 32) >> 4;
                        mma_ss(acc, dA_ + offa, dS + offs, iOutK, (s & 1) || k > 0);
                    }
                }
                mma_commit(&sm->mma_a);
                iss_a = true;
            }
        }
        __syncwarp();

        // masks, one 32-column group J of the row at a time (J = 2 half, 2 half + 1):
        //   M^T_ti = 2^(c_i - c_t) dt_t K_ti and V^T_ti = 2^(c_i - c_t) dt_t Z^T_ti  (i >= t)
        //   V_tj   = 2^(c_t - c_j) dt_j Z_tj                                     (j <= t)
        // with the row sums a_t = sum_i 2^(c_i - c_t) K_ti Z^T_ti and the column
        // sums of M^T o Z^T (transposed across the warp)
        float acc_a = 0.f;
        // one verdict per warp: the transpose sums below shuffle across all lanes
        const bool ok = __all_sync(0xffffffffu, wait_bounded(&sm->mma_a, ph, ab, a.err, a.wait, kErrBwdMma));
        tc_fence_after();
#pragma unroll 1
        for (int J = 2 * half; J < 2 * half + 2; ++J) {
            float prod[32];
            {
                uint32_t pk[16], pl[16], qk[16], ql[16];
                if (J < q || !ok) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) prod[k] = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = pl[k] = qk[k] = ql[k] = 0u;
                } else {
                    uint32_t kk[32], zz[32];
                    tmem_ld32(tmem + lane_base + 32 * J, kk);
                    tmem_ld32(tmem + lane_base + 128 + 32 * J, zz);
                    tmem_wait_ld();
                    reg_fence32(kk);
                    reg_fence32(zz);
                    float wv[32];
                    if (mono && J > q) {
                        const float rT = fast_exp2(sm->c2[32 * J] - c2t);
#pragma unroll
                        for (int k = 0; k < 32; ++k) wv[k] = sm->colT[32 * J + k] * rT;
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const bool keep = (J > q) || (k >= lane);  // i >= t
                            wv[k] = keep ? fast_exp2(sm->c2[32 * J + k] - c2t) : 0.f;
                        }
                    }
                    const f2 dt2 = f2_pack(dtt, dtt);
                    f2 a2 = f2_pack(0.f, 0.f);
                    float m[32], vt[32];
#pragma unroll
                    for (int k = 0; k < 32; k += 2) {
                        const f2 w2 = f2_pack(wv[k], wv[k + 1]);
                        const f2 zv = f2_pack(__uint_as_float(zz[k]), __uint_as_float(zz[k + 1]));
                        const f2 wk = f2_mul(w2, f2_pack(__uint_as_float(kk[k]), __uint_as_float(kk[k + 1])));
                        a2 = f2_fma(wk, zv, a2);
                        const f2 mk = f2_mul(wk, dt2);
                        f2_unpack(mk, m[k], m[k + 1]);
                        f2_unpack(f2_mul(mk, zv), prod[k], prod[k + 1]);
                        f2_unpack(f2_mul(f2_mul(w2, dt2), zv), vt[k], vt[k + 1]);
                    }
                    float a0, a1;
                    f2_unpack(a2, a0, a1);
                    acc_a += a0 + a1;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        split_bf16x2(m[2 * k], m[2 * k + 1], pk[k], pl[k]);
                        split_bf16x2(vt[2 * k], vt[2 * k + 1], qk[k], ql[k]);
                    }
                }
                tmem_st16(tmem + lane_base + 32 * J, pk);
                tmem_st16(tmem + lane_base + 32 * J + 16, pl);
                tmem_st16(tmem + lane_base + 128 + 32 * J, qk);
                tmem_st16(tmem + lane_base + 128 + 32 * J + 16, ql);
            }
            sm->spart[q][32 * J + lane] = transpose_sum32(prod);
            {
                uint32_t pk[16], pl[16];
                if (J > q || !ok) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = pl[k] = 0u;
                } else {
                    uint32_t z[32];
                    tmem_ld32(tmem + lane_base + 256 + 32 * J, z);
                    tmem_wait_ld();
                    reg_fence32(z);
                    float v[32];
                    if (mono && J < q) {
                        const f2 r2 = f2_pack(fast_exp2(c2t - sm->c2[32 * q]), fast_exp2(c2t - sm->c2[32 * q]));
#pragma unroll
                        for (int k = 0; k < 32; k += 2)
                            f2_unpack(f2_mul(f2_mul(r2, f2_pack(sm->colV[q][32 * J + k], sm->colV[q][32 * J + k + 1])),
                                             f2_pack(__uint_as_float(z[k]), __uint_as_float(z[k + 1]))),
                                      v[k], v[k + 1]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int j = 32 * J + k;
                            const bool lowr = (J < q) || (k <= lane);  // j <= t
                            v[k] = lowr ? fast_exp2(c2t - sm->c2[j]) * sm->dt[j] * __uint_as_float(z[k]) : 0.f;
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) split_bf16x2(v[2 * k], v[2 * k + 1], pk[k], pl[k]);
                }
                tmem_st16(tmem + lane_base + 256 + 32 * J, pk);
                tmem_st16(tmem + lane_base + 256 + 32 * J + 16, pl);
            }
        }
        sm->part[0][half][t] = acc_a;

        // token sums over this half's 32 head-dim columns: X_t.BR_t, dY_t.CH_t,
        // dY_t.X_t (C H^T is read before dX takes its columns)
        const bool tiles = wait_bounded(&sm->full, ph, ab, a.err, a.wait, kErrBwdLoad);
        float xv[32], yv[32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint4 ux = make_uint4(0, 0, 0, 0), uy = ux;
            if (tiles) {
                ux = *reinterpret_cast<const uint4 *>(smem + oMX + swz(t, 4 * half + cc));
                uy = *reinterpret_cast<const uint4 *>(smem + oMdY + swz(t, 4 * half + cc));
            }
            const uint32_t wx[4] = {ux.x, ux.y, ux.z, ux.w}, wy[4] = {uy.x, uy.y, uy.z, uy.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                xv[8 * cc + 2 * k] = bf16_lo(wx[k]);
                xv[8 * cc + 2 * k + 1] = bf16_hi(wx[k]);
                yv[8 * cc + 2 * k] = bf16_lo(wy[k]);
                yv[8 * cc + 2 * k + 1] = bf16_hi(wy[k]);
            }
        }
        float xbr = 0.f, ych = 0.f, yx = 0.f;
        if (ok) {
            uint32_t br[32], ch[32];
            tmem_ld32(tmem + lane_base + 384 + 32 * half, br);
            tmem_ld32(tmem + lane_base + 448 + 32 * half, ch);
            tmem_wait_ld();
            reg_fence32(br);
            reg_fence32(ch);
            f2 xb2 = f2_pack(0.f, 0.f), yc2 = xb2;
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                xb2 = f2_fma(f2_pack(xv[k], xv[k + 1]),
                             f2_pack(__uint_as_float(br[k]), __uint_as_float(br[k + 1])), xb2);
                yc2 = f2_fma(f2_pack(yv[k], yv[k + 1]),
                             f2_pack(__uint_as_float(ch[k]), __uint_as_float(ch[k + 1])), yc2);
            }
            float s0, s1;
            f2_unpack(xb2, s0, s1);
            xbr = s0 + s1;
            f2_unpack(yc2, s0, s1);
            ych = s0 + s1;
        }
        {
            f2 yx2 = f2_pack(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 32; k += 2)
                yx2 = f2_fma(f2_pack(yv[k], yv[k + 1]), f2_pack(xv[k], xv[k + 1]), yx2);
            float s0, s1;
            f2_unpack(yx2, s0, s1);
            yx = s0 + s1;
        }
        sm->part[1][half][t] = xbr;
        sm->part[2][half][t] = ych;
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();

        // dX = M^T dY into the C H^T columns: A = M^T from TMEM (hi groups, then
        // lo), B = dY MN-major
        if (tid == 0 && ok && !*(volatile int *)ab) {
            tc_fence_after();
            const uint64_t ddYmn = sdesc_sw128(base + oMdY, 1024, 1024);
#pragma unroll
            for (int k = 0; k < kQ / 16; ++k)
                mma_ts(tmem + 448, tmem + 32 * (k >> 1) + 8 * (k & 1), ddYmn + ((k * 2048) >> 4), iDiag, k > 0);
#pragma unroll
            for (int k = 0; k < kQ / 16; ++k)
                mma_ts(tmem + 448, tmem + 32 * (k >> 1) + 16 + 8 * (k & 1), ddYmn + ((k * 2048) >> 4), iDiag, 1);
            mma_commit(&sm->mma_b);
            iss_b = true;
        }

        // the row's totals, the same in both halves
        acc_a = sm->part[0][0][t] + sm->part[0][1][t];
        xbr = sm->part[1][0][t] + sm->part[1][1][t];
        ych = sm->part[2][0][t] + sm->part[2][1][t];
        const float e_t = fast_exp2(c2t);
        const float dec_t = fast_exp2(tot2 - c2t);
        const float u_t = dec_t * dtt;
        const float s_row = sm->spart[0][t] + sm->spart[1][t] + sm->spart[2][t] + sm->spart[3][t];
        const float dcum = s_row - dtt * acc_a + e_t * ych - u_t * xbr;
        // in one exchange: sum_j u_j X_j.BR_j, <R, H>, dY.X and sum_t dcum_t
        // (row values counted by half 0 only: half 1 holds the same), and the
        // per-half prefix of dcum. The last token's dcum gains
        // 2^tot <R, H> + sum_j u_j X_j.BR_j, which enters every row's suffix sum.
        float pre;
        const float4 tots = block_sums_row_scan256(
            make_float4(half == 0 ? u_t * xbr : 0.f, rh_dot, yx, half == 0 ? dcum : 0.f), dcum,
            pre, sm->red5);
        const float extra = fast_exp2(tot2) * tots.y + tots.x;
        const float sdc = tots.w - pre + dcum + extra;  // sum over tokens k >= t
        const float ddt_t = acc_a + dec_t * xbr + Ah * sdc;
        const float dA_c = block_sum256(half == 0 ? dtt * sdc : 0.f, sm->red);
        const float dD_c = tots.z;
        const bool fine = ok && !*(volatile int *)ab;
        if (fine && half == 0 && t < n) a.ddt[((long long)b * a.L + t0 + t) * a.H + h] = ddt_t;
        if (fine && tid == 0) {
            a.dA_part[lane_bh * a.nc + c] = dA_c;
            a.dD_part[lane_bh * a.nc + c] = dD_c;
        }

        // dx_t = D dY_t + dX_t + u_t BR_t, this half's 32 columns, as row t of a
        // 128 x 32 fp32 tile (128-byte swizzle), then one bulk tensor store per
        // half; the store skips rows past the sequence's end
        const bool ok2 = ok && wait_bounded(&sm->mma_b, ph, ab, a.err, a.wait, kErrBwdMma);
        tc_fence_after();
        if (ok2) {
            uint32_t acc[32], br[32];
            tmem_ld32(tmem + lane_base + 448 + 32 * half, acc);
            tmem_ld32(tmem + lane_base + 384 + 32 * half, br);
            tmem_wait_ld();
            reg_fence32(acc);
            reg_fence32(br);
            unsigned char *dxs = smem + oMDX + half * kTile;
            const f2 D2 = f2_pack(Dh, Dh), u2 = f2_pack(u_t, u_t);
            auto dx2 = [&](int k) {
                return f2_fma(D2, f2_pack(yv[k], yv[k + 1]),
                              f2_fma(u2, f2_pack(__uint_as_float(br[k]), __uint_as_float(br[k + 1])),
                                     f2_pack(__uint_as_float(acc[k]), __uint_as_float(acc[k + 1]))));
            };
#pragma unroll
            for (int k = 0; k < 32; k += 4)
                *reinterpret_cast<ulonglong2 *>(dxs + swz(t, k >> 2)) = make_ulonglong2(dx2(k), dx2(k + 2));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();  // dX and B R^T read: columns 0-127 and 384-511 free

        // dB = V^T C (A = V^T from TMEM, B = C MN-major) into 0-127, X R into
        // 384-511; dx leaves meanwhile
        const uint64_t dCt = sdesc_sw128(base + oMC, kTile, 1024);
        const uint64_t dBt = sdesc_sw128(base + oMB, kTile, 1024);
        if (tid == 0) {
            if (ok2 && !*(volatile int *)ab) {
                tma_store_4d(&mDX, smem + oMDX, 0, h, t0, b);
                tma_store_4d(&mDX, smem + oMDX + kTile, 32, h, t0, b);
                bulk_commit();
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kQ / 16; ++k)
                    mma_ts(tmem + 0, tmem + 128 + 32 * (k >> 1) + 8 * (k & 1), dCt + ((k * 2048) >> 4), iWideMN, k > 0);
#pragma unroll
                for (int k = 0; k < kQ / 16; ++k)
                    mma_ts(tmem + 0, tmem + 128 + 32 * (k >> 1) + 16 + 8 * (k & 1), dCt + ((k * 2048) >> 4), iWideMN, 1);
                const uint64_t dRh = sdesc_sw128(base + oMRh, kHalfTile, 1024);
                const uint64_t dRl = sdesc_sw128(base + oMRl, kHalfTile, 1024);
#pragma unroll
                for (int k = 0; k < kP / 16; ++k)
                    mma_ss(tmem + 384, dX + ((k * 32) >> 4), dRh + ((k * 2048) >> 4), iWideMN, k > 0);
#pragma unroll
                for (int k = 0; k < kP / 16; ++k)
                    mma_ss(tmem + 384, dX + ((k * 32) >> 4), dRl + ((k * 2048) >> 4), iWideMN, 1);
                mma_commit(&sm->mma_c);
                iss_c = true;
            }
        }
        // dB_j = (V^T C)_j + u_j (X R)_j, column group J as row t of the 128 x 32
        // fp32 tile J where C and R were (their MMAs are done)
        const bool okc = ok2 && wait_bounded(&sm->mma_c, ph, ab, a.err, a.wait, kErrBwdMma);
        tc_fence_after();
#pragma unroll 1
        for (int J = 2 * half; J < 2 * half + 2; ++J) {
            uint32_t acc[32], xr[32];
            tmem_ld32(tmem + lane_base + 0 + 32 * J, acc);
            tmem_ld32(tmem + lane_base + 384 + 32 * J, xr);
            tmem_wait_ld();
            reg_fence32(acc);
            reg_fence32(xr);
            if (okc) {
                unsigned char *stg = smem + oMC + J * kTile;
                const f2 u2 = f2_pack(u_t, u_t);
                auto db2 = [&](int k) {
                    return f2_fma(u2, f2_pack(__uint_as_float(xr[k]), __uint_as_float(xr[k + 1])),
                                  f2_pack(__uint_as_float(acc[k]), __uint_as_float(acc[k + 1])));
                };
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    *reinterpret_cast<ulonglong2 *>(stg + swz(t, k >> 2)) = make_ulonglong2(db2(k), db2(k + 2));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();  // dB staged; columns 0-127 and 384-511 free again

        // dC = V B (A = V from TMEM) into 128-255, dY H into 384-511; then the dB
        // tiles are added into the group's dB in L2 (one bulk tensor reduction per
        // 32 columns; rows past the sequence's end are skipped)
        if (tid == 0 && okc && !*(volatile int *)ab) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kQ / 16; ++k)
                mma_ts(tmem + 128, tmem + 256 + 32 * (k >> 1) + 8 * (k & 1), dBt + ((k * 2048) >> 4), iWideMN, k > 0);
#pragma unroll
            for (int k = 0; k < kQ / 16; ++k)
                mma_ts(tmem + 128, tmem + 256 + 32 * (k >> 1) + 16 + 8 * (k & 1), dBt + ((k * 2048) >> 4), iWideMN, 1);
            const uint64_t dHh = sdesc_sw128(base + oMHh, kHalfTile, 1024);
            const uint64_t dHl = sdesc_sw128(base + oMHl, kHalfTile, 1024);
#pragma unroll
            for (int k = 0; k < kP / 16; ++k)
                mma_ss(tmem + 384, ddY + ((k * 32) >> 4), dHh + ((k * 2048) >> 4), iWideMN, k > 0);
#pragma unroll
            for (int k = 0; k < kP / 16; ++k)
                mma_ss(tmem + 384, ddY + ((k * 32) >> 4), dHl + ((k * 2048) >> 4), iWideMN, 1);
            mma_commit(&sm->mma_d);
            iss_d = true;
#pragma unroll
            for (int J = 0; J < 4; ++J) tma_reduce_add_4d(&mDB, smem + oMC + J * kTile, 32 * J, g, t0, b);
            bulk_commit();
        }
        // dC_i = (V B)_i + e_i (dY H)_i, staged where X, dY and B were
        const bool okd = okc && wait_bounded(&sm->mma_d, ph, ab, a.err, a.wait, kErrBwdMma);
        tc_fence_after();
#pragma unroll 1
        for (int J = 2 * half; J < 2 * half + 2; ++J) {
            uint32_t acc[32], yh[32];
            tmem_ld32(tmem + lane_base + 128 + 32 * J, acc);
            tmem_ld32(tmem + lane_base + 384 + 32 * J, yh);
            tmem_wait_ld();
            reg_fence32(acc);
            reg_fence32(yh);
            if (okd) {
                unsigned char *stg = smem + J * kTile;
                const f2 e2 = f2_pack(e_t, e_t);
                auto dc2 = [&](int k) {
                    return f2_fma(e2, f2_pack(__uint_as_float(yh[k]), __uint_as_float(yh[k + 1])),
                                  f2_pack(__uint_as_float(acc[k]), __uint_as_float(acc[k + 1])));
                };
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                    *reinterpret_cast<ulonglong2 *>(stg + swz(t, k >> 2)) = make_ulonglong2(dc2(k), dc2(k + 2));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            if (okd && !*(volatile int *)ab) {
#pragma unroll
                for (int J = 0; J < 4; ++J) tma_reduce_add_4d(&mDC, smem + J * kTile, 32 * J, g, t0, b);
                bulk_commit();
            }
            bulk_wait_read0();  // the stores and reductions have read their tiles
        }
        // after an abort, loads or MMAs may still be in flight: wait for each
        // (bounded) before TMEM is freed and the CTA exits
        if (tid == 0 && *(volatile int *)ab) {
            mbar_wait(&sm->full, ph, kWait);
            if (iss_a) mbar_wait(&sm->mma_a, ph, kWait);
            if (iss_b) mbar_wait(&sm->mma_b, ph, kWait);
            if (iss_c) mbar_wait(&sm->mma_c, ph, kWait);
            if (iss_d) mbar_wait(&sm->mma_d, ph, kWait);
        }
        // the item's TMEM reads, tile reads and staged outputs are done: the next
        // item may load and overwrite them (the flag is stable past this barrier)
        tc_fence_before();
        __syncthreads();
        if (*(volatile int *)ab) break;
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// The chunk states chained along a lane in one pass. Each chunk's own
// contribution is, for the forward chain,
//   S_c = sum_j 2^(tot - c_j) dt_j x_j (x) B_j
// or, with ADJ, its contribution to its entering state's gradient
//   G_c = sum_i 2^(c_i) dy_i (x) C_i        (x := dy, B := C)
// as S^T = B^T (w o X) on the tensor cores (the forward's chunk-state MMA:
// w o X as bf16 hi | lo side by side, 128 output columns summed in pairs).
// One CTA per (batch, head) lane walks its chunks in order and carries the
// running value in registers (thread n holds row n of it, N x P as the MMA
// leaves it in TMEM):
//   forward, chunk 0 up:      out[c] = H, then H <- 2^tot_c H + S_c   (H = h0 at first)
//   ADJ, last chunk down:     out[c] = R, then R <- 2^tot_c R + G_c   (R = dh_final at
//                             first; dh0 = R after chunk 0)
// so the per-chunk contributions never go through memory: the chain is
// written once per chunk (a per-chunk kernel writing S and a separate pass
// reading it and writing the chain took 237 us against 147 us, 243 against
// 153 for the adjoint, on the 2.7B-style layer). The next chunk's tiles are
// requested as soon as this chunk's MMA has read them, its steps one chunk
// ahead. w o X hi is written over X (each thread rewrites only its own row),
// so that three CTAs fit on an SM.
constexpr int o3X = 0, o3B = kTile, o3Wl = 3 * kTile, o3Small = 4 * kTile;

struct Small3 {
    float scan[kQ];
    float tot;
    uint64_t full, mma;
    uint32_t tmem_base;
    int abort;
};
constexpr int smem3_bytes() { return o3Small + (int)sizeof(Small3) + 1024; }
static_assert(3 * smem3_bytes() <= 227 * 1024, "three CTAs per SM");

// For few lanes the chains leave SMs idle (at b1 H80, 80 lanes: 52 us each
// against 20 us for a per-chunk launch), so the chunk states are also formed
// one CTA per (chunk, head, batch), three per SM, written to memory for the
// CUDA-core state passes:
//   S_c (or G_c) as above, out (lanes, nc, P, N) fp32, and decay = 2^tot.
struct Bwd3Args {
    const __nv_bfloat16 *dt;
    const float *A;
    float *S, *decay;
    unsigned int *err;
    long long wait;  // bound of each wait, clock cycles
    int L, H, G, nc;
};

template <bool ADJ>
__global__ void __launch_bounds__(kThreads, 3)
tc_bwd_states_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mB,
                     const Bwd3Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Small3 *sm = reinterpret_cast<Small3 *>(smem + o3Small);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.H / a.G);
    const int t = threadIdx.x, warp = t >> 5;
    const int t0 = c * kQ;
    const int n = min(kQ, a.L - t0);
    const long long lane_bh = (long long)b * a.H + h;
    const float Ah = a.A[h];

    if (t == 0) {
        mbar_init(&sm->full, 1);
        mbar_init(&sm->mma, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    int *ab = &sm->abort;
    bool iss = false;

    if (t == 0) {
        mbar_arrive_expect_tx(&sm->full, 3 * kTile);
        tma_load_4d(smem + o3X, &mX, &sm->full, 0, h, t0, b);
        tma_load_4d(smem + o3B, &mB, &sm->full, 0, g, t0, b);
        tma_load_4d(smem + o3B + kTile, &mB, &sm->full, 64, g, t0, b);
    }
    const float dtt = t < n ? __bfloat162float(a.dt[((long long)b * a.L + t0 + t) * a.H + h]) : 0.f;
    const float c2t = block_scan128(dtt * Ah * kLog2e, sm->scan);
    if (t == kQ - 1) sm->tot = c2t;
    __syncthreads();
    const float tot2 = sm->tot;
    const float wt = ADJ ? fast_exp2(c2t) : fast_exp2(tot2 - c2t) * dtt;

    // row t of w o X as bf16 hi + lo
    const bool tiles = wait_bounded(&sm->full, 0, ab, a.err, a.wait, kErrBwdLoad);
    if (tiles) {
#pragma unroll 2
        for (int cc = 0; cc < 8; ++cc) {
            const uint32_t off = swz(t, cc);
            const uint4 u = *reinterpret_cast<const uint4 *>(smem + o3X + off);
            const uint32_t xw[4] = {u.x, u.y, u.z, u.w};
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float v0 = wt * bf16_lo(xw[k]), v1 = wt * bf16_hi(xw[k]);
                split_bf16x2(v0, v1, hw[k], lw[k]);
            }
            *reinterpret_cast<uint4 *>(smem + o3X + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(smem + o3Wl + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0 && tiles && !*(volatile int *)ab) {
        tc_fence_after();
        constexpr uint32_t iState2 = idesc_bf16(128, 128, true, true);
        const uint32_t base = smem_u32(smem);
        const uint64_t dbt = sdesc_sw128(base + o3B, kTile, 1024);          // B^T, M = state
        const uint64_t dw2 = sdesc_sw128(base + o3X, o3Wl - o3X, 1024);     // hi | lo
#pragma unroll
        for (int k = 0; k < kQ / 16; ++k)
            mma_ss(tmem, dbt + ((k * 2048) >> 4), dw2 + ((k * 2048) >> 4), iState2, k > 0);
        mma_commit(&sm->mma);
        iss = true;
    }
    const bool ok = tiles && wait_bounded(&sm->mma, 0, ab, a.err, a.wait, kErrBwdMma);
    tc_fence_after();
    // thread t = state index: S[p][t] = hi[p] + lo[p]
    float *Sp = a.S + (lane_bh * a.nc + c) * (long long)kP * kN;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        uint32_t hi[32], lo[32];
        tmem_ld32(tmem + lane_base + 32 * half, hi);
        tmem_ld32(tmem + lane_base + 64 + 32 * half, lo);
        tmem_wait_ld();
        reg_fence32(hi);
        reg_fence32(lo);
        if (ok && !*(volatile int *)ab) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
                Sp[(long long)(32 * half + k) * kN + t] = __uint_as_float(hi[k]) + __uint_as_float(lo[k]);
        }
    }
    if (t == 0 && ok) a.decay[lane_bh * a.nc + c] = fast_exp2(tot2);
    if (t == 0 && *(volatile int *)ab) {
        mbar_wait(&sm->full, 0, kWait);
        if (iss) mbar_wait(&sm->mma, 0, kWait);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

struct BwdCArgs {
    const __nv_bfloat16 *dt;
    const float *A;
    const float *init;  // h0 or dh_final, (lanes, P, N), or null (zero)
    float *out;         // (lanes, nc, P, N)
    float *final_out;   // ADJ: dh0 (lanes, P, N), or null
    unsigned int *err;
    long long wait;     // bound of each wait, clock cycles
    int L, H, G, nc;
};

template <bool ADJ>
__global__ void __launch_bounds__(kThreads, 3)
tc_bwd_chain_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mB,
                    const BwdCArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Small3 *sm = reinterpret_cast<Small3 *>(smem + o3Small);
    const long long lane_bh = blockIdx.x;
    const int h = (int)(lane_bh % a.H), b = (int)(lane_bh / a.H);
    const int g = h / (a.H / a.G);
    const int t = threadIdx.x, warp = t >> 5;
    const long long PN = (long long)kP * kN;
    const float Ah = a.A[h];

    if (t == 0) {
        mbar_init(&sm->full, 1);
        mbar_init(&sm->mma, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const uint32_t base = smem_u32(smem);
    int *ab = &sm->abort;

    auto chunk_of = [&](int i) { return ADJ ? a.nc - 1 - i : i; };
    auto issue = [&](int c) {  // thread 0: chunk c's X (or dY) and B (or C) tiles
        const int t0 = c * kQ;
        mbar_arrive_expect_tx(&sm->full, 3 * kTile);
        tma_load_4d(smem + o3X, &mX, &sm->full, 0, h, t0, b);
        tma_load_4d(smem + o3B, &mB, &sm->full, 0, g, t0, b);
        tma_load_4d(smem + o3B + kTile, &mB, &sm->full, 64, g, t0, b);
    };
    auto load_dt = [&](int c) -> float {
        const int tok = c * kQ + t;
        return tok < a.L ? __bfloat162float(a.dt[((long long)b * a.L + tok) * a.H + h]) : 0.f;
    };

    // the running value: this thread's state row n = t, p = 0..63
    float hv[kP];
    {
        const float *in = a.init ? a.init + lane_bh * PN : nullptr;
#pragma unroll
        for (int k = 0; k < kP; ++k) hv[k] = in ? __ldcg(in + (long long)k * kN + t) : 0.f;
    }
    int pend_full = -1, pend_mma = -1;  // thread 0: the iteration whose copy / MMA is in flight
    if (t == 0) {
        tma_prefetch_desc(&mX);
        issue(chunk_of(0));
        pend_full = 0;
    }
    float dt_next = load_dt(chunk_of(0));
#pragma unroll 1
    for (int i = 0; i < a.nc; ++i) {
        const int c = chunk_of(i);
        const uint32_t ph = i & 1;
        const float dtt = dt_next;
        if (i + 1 < a.nc) dt_next = load_dt(chunk_of(i + 1));
        const float c2t = block_scan128(dtt * Ah * kLog2e, sm->scan);
        if (t == kQ - 1) sm->tot = c2t;
        __syncthreads();
        const float tot2 = sm->tot;
        const float wt = ADJ ? fast_exp2(c2t) : fast_exp2(tot2 - c2t) * dtt;

        // row t of w o X as bf16 hi (over X) + lo
        const bool tiles = wait_bounded(&sm->full, ph, ab, a.err, a.wait, kErrBwdLoad);
        if (t == 0 && tiles) pend_full = -1;
        if (tiles) {
#pragma unroll 2
            for (int cc = 0; cc < 8; ++cc) {
                const uint32_t off = swz(t, cc);
                const uint4 u = *reinterpret_cast<const uint4 *>(smem + o3X + off);
                const uint32_t xw[4] = {u.x, u.y, u.z, u.w};
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float v0 = wt * bf16_lo(xw[k]), v1 = wt * bf16_hi(xw[k]);
                    split_bf16x2(v0, v1, hw[k], lw[k]);
                }
                *reinterpret_cast<uint4 *>(smem + o3X + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(smem + o3Wl + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (t == 0 && tiles && !*(volatile int *)ab) {
            tc_fence_after();
            constexpr uint32_t iState2 = idesc_bf16(128, 128, true, true);
            const uint64_t dbt = sdesc_sw128(base + o3B, kTile, 1024);       // B^T, M = state
            const uint64_t dw2 = sdesc_sw128(base + o3X, o3Wl - o3X, 1024);  // hi | lo
#pragma unroll
            for (int k = 0; k < kQ / 16; ++k)
                mma_ss(tmem, dbt + ((k * 2048) >> 4), dw2 + ((k * 2048) >> 4), iState2, k > 0);
            mma_commit(&sm->mma);
            pend_mma = i;
        }
        const bool ok = tiles && wait_bounded(&sm->mma, ph, ab, a.err, a.wait, kErrBwdMma);
        tc_fence_after();
        if (t == 0 && ok) {
            pend_mma = -1;
            // the tiles are read: the next chunk's go out now
            if (i + 1 < a.nc && !*(volatile int *)ab) {
                issue(chunk_of(i + 1));
                pend_full = i + 1;
            }
        }

        // out[c] = the running value, then its update with this chunk's
        // decay and contribution (hi + lo columns)
        float *op = a.out + (lane_bh * a.nc + c) * PN;
        const float dc = fast_exp2(tot2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // unrolled: hv stays in registers
            uint32_t hi[32], lo[32];
            tmem_ld32(tmem + lane_base + 32 * half, hi);
            tmem_ld32(tmem + lane_base + 64 + 32 * half, lo);
            tmem_wait_ld();
            reg_fence32(hi);
            reg_fence32(lo);
            if (ok) {
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int p = 32 * half + k;
                    op[(long long)p * kN + t] = hv[p];
                    hv[p] = fmaf(dc, hv[p], __uint_as_float(hi[k]) + __uint_as_float(lo[k]));
                }
            }
        }
        // TMEM and the decay read before the next chunk's MMA and scan
        tc_fence_before();
        __syncthreads();
        if (*(volatile int *)ab) break;
    }
    if (ADJ && a.final_out && !*(volatile int *)ab) {
        float *fo = a.final_out + lane_bh * PN;
#pragma unroll
        for (int k = 0; k < kP; ++k) fo[(long long)k * kN + t] = hv[k];
    }
    // after an abort, a copy or MMA may still be in flight: wait for it
    // (bounded) before TMEM is freed and the CTA exits
    if (t == 0 && *(volatile int *)ab) {
        if (pend_full >= 0) mbar_wait(&sm->full, pend_full & 1, kWait);
        if (pend_mma >= 0) mbar_wait(&sm->mma, pend_mma & 1, kWait);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode_bwd = nullptr;

int bwd_num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

ssd_status bwd_encoder() {
    if (!g_encode_bwd) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_bwd = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!g_encode_bwd) return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    return SSD_OK;
}

// bf16 (d3, d2, d1, d0) row-major, box {64, 1, 128, 1}, 128-byte swizzle, zero fill
ssd_status bwd_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint64_t d3) {
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kQ, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = g_encode_bwd(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
                                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SSD_OK;
}

// fp32 (d3, d2, d1, d0) row-major, box {32, 1, 128, 1}, 128-byte swizzle: the
// staged output tiles (dx, and dB and dC added in by bulk tensor reductions)
ssd_status bwd_map_f32(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t d3) {
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 4, d0 * d1 * 4, d0 * d1 * d2 * 4};
    const cuuint32_t box[4] = {32, 1, (cuuint32_t)kQ, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = g_encode_bwd(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void *>(base),
                                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SSD_OK;
}

}  // namespace

// Per-chunk states of 128-token chunks on the tensor cores: S (lanes, nc, P,
// N) and decay (lanes, nc) as chunk_states_launch gives them for chunk 128.
ssd_status tc_chunk_states(const Problem &pr, const void *x, const void *dt, const float *A,
                           const void *B, float *S, float *decay, bool adjoint, cudaStream_t st) {
    ssd_status s;
    if ((s = bwd_encoder()) != SSD_OK) return s;
    const uint64_t L = (uint64_t)pr.seqlen, H = (uint64_t)pr.nheads, G = (uint64_t)pr.ngroups;
    const uint64_t bt = (uint64_t)pr.batch;
    CUtensorMap mX, mB;
    if ((s = bwd_map(&mX, x, kP, H, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map(&mB, B, kN, G, L, bt)) != SSD_OK) return s;
    const int nc = (int)((pr.seqlen + kQ - 1) / kQ);
    if (nc == 0) return SSD_OK;
    Bwd3Args a3;
    a3.dt = static_cast<const __nv_bfloat16 *>(dt);
    a3.A = A;
    a3.S = S;
    a3.decay = decay;
    a3.err = device_error_word();
    a3.wait = wait_limit_cycles();
    a3.L = (int)L;
    a3.H = (int)H;
    a3.G = (int)G;
    a3.nc = nc;
    const dim3 grid((unsigned)nc, (unsigned)H, (unsigned)bt);
    cudaError_t e;
    if (adjoint) {
        if ((e = cudaFuncSetAttribute(tc_bwd_states_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem3_bytes())) != cudaSuccess)
            return cuda_fail(e, "tc_bwd_states smem");
        launch_begin("tc_bwd_adjoint_states", st);
        tc_bwd_states_kernel<true><<<grid, kThreads, smem3_bytes(), st>>>(mX, mB, a3);
    } else {
        if ((e = cudaFuncSetAttribute(tc_bwd_states_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem3_bytes())) != cudaSuccess)
            return cuda_fail(e, "tc_bwd_states smem");
        launch_begin("tc_bwd_chunk_states", st);
        tc_bwd_states_kernel<false><<<grid, kThreads, smem3_bytes(), st>>>(mX, mB, a3);
    }
    launch_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tc_bwd_states launch");
    return SSD_OK;
}

// The chunk states chained along each lane in one pass (see tc_bwd_chain_kernel):
// out = the state entering each 128-token chunk (from init = h0), or with
// adjoint the gradient at each chunk's end (from init = dh_final) and
// final_out = dh0; both (lanes, nc, P, N) fp32.
ssd_status tc_state_chain(const Problem &pr, const void *x, const void *dt, const float *A,
                          const void *B, const float *init, float *out, float *final_out,
                          bool adjoint, cudaStream_t st) {
    ssd_status s;
    if ((s = bwd_encoder()) != SSD_OK) return s;
    const uint64_t L = (uint64_t)pr.seqlen, H = (uint64_t)pr.nheads, G = (uint64_t)pr.ngroups;
    const uint64_t bt = (uint64_t)pr.batch;
    CUtensorMap mX, mB;
    if ((s = bwd_map(&mX, x, kP, H, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map(&mB, B, kN, G, L, bt)) != SSD_OK) return s;
    const int nc = (int)((pr.seqlen + kQ - 1) / kQ);
    if (nc == 0) return SSD_OK;
    BwdCArgs ac;
    ac.dt = static_cast<const __nv_bfloat16 *>(dt);
    ac.A = A;
    ac.init = init;
    ac.out = out;
    ac.final_out = final_out;
    ac.err = device_error_word();
    ac.wait = wait_limit_cycles();
    ac.L = (int)L;
    ac.H = (int)H;
    ac.G = (int)G;
    ac.nc = nc;
    const dim3 grid((unsigned)(bt * H));
    cudaError_t e;
    if (adjoint) {
        if ((e = cudaFuncSetAttribute(tc_bwd_chain_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem3_bytes())) != cudaSuccess)
            return cuda_fail(e, "tc_bwd_chain smem");
        launch_begin("tc_bwd_adjoint_chain", st);
        tc_bwd_chain_kernel<true><<<grid, kThreads, smem3_bytes(), st>>>(mX, mB, ac);
    } else {
        if ((e = cudaFuncSetAttribute(tc_bwd_chain_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem3_bytes())) != cudaSuccess)
            return cuda_fail(e, "tc_bwd_chain smem");
        launch_begin("tc_bwd_state_chain", st);
        tc_bwd_chain_kernel<false><<<grid, kThreads, smem3_bytes(), st>>>(mX, mB, ac);
    }
    launch_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tc_bwd_chain launch");
    return SSD_OK;
}

// The chains walk one lane per CTA, three per SM: with fewer lanes than two
// SMs' worth they leave SMs idle, and per-chunk CTAs with separate state
// passes finish sooner.
bool tc_chain_pays(const Problem &pr) {
    return pr.batch * pr.nheads >= 2LL * bwd_num_sms();
}

// The tensor-core path takes bf16 I/O with P = 64, N = 128 (128-token chunks).
bool tc_backward_supported(const Problem &pr) {
    return pr.dtype == SSD_BF16 && pr.headdim == kP && pr.dstate == kN && pr.seqlen > 0;
}

// Per-chunk gradients from the states entering each 128-token chunk (Hst) and
// the gradients at each chunk's end (R), both (lanes, nc, P, N) fp32: dx, ddt,
// dB and dC (added into the caller's zeroed arrays), and the per-(lane, chunk)
// parts of dA and dD.
ssd_status tc_backward_chunks(const Problem &pr, const void *x, const void *dt, const float *A,
                              const void *B, const void *C, const float *D, const void *dy,
                              const float *Hst, const float *R, float *dx, float *ddt, float *dB,
                              float *dC, float *dA_part, float *dD_part, cudaStream_t st) {
    ssd_status s;
    if ((s = bwd_encoder()) != SSD_OK) return s;
    const uint64_t L = (uint64_t)pr.seqlen, H = (uint64_t)pr.nheads, G = (uint64_t)pr.ngroups;
    const uint64_t bt = (uint64_t)pr.batch;
    CUtensorMap mX, mdY, mB, mC;
    if ((s = bwd_map(&mX, x, kP, H, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map(&mdY, dy, kP, H, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map(&mB, B, kN, G, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map(&mC, C, kN, G, L, bt)) != SSD_OK) return s;
    CUtensorMap mDX, mDB, mDC;
    if ((s = bwd_map_f32(&mDX, dx, kP, H, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map_f32(&mDB, dB, kN, G, L, bt)) != SSD_OK) return s;
    if ((s = bwd_map_f32(&mDC, dC, kN, G, L, bt)) != SSD_OK) return s;
    const int nc = (int)((pr.seqlen + kQ - 1) / kQ);
    const dim3 grid((unsigned)nc, (unsigned)H, (unsigned)bt);
    unsigned int *err = device_error_word();
    cudaError_t e;

    BwdMArgs am;
    am.dt = static_cast<const __nv_bfloat16 *>(dt);
    am.A = A;
    am.D = D;
    am.Hst = Hst;
    am.Rst = R;
    am.ddt = ddt;
    am.dA_part = dA_part;
    am.dD_part = dD_part;
    am.err = err;
    am.wait = wait_limit_cycles();
    am.L = (int)L;
    am.H = (int)H;
    am.G = (int)G;
    am.nc = nc;
    am.batch = (int)bt;
    if ((e = cudaFuncSetAttribute(tc_bwd_chunk_grads_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smemM_bytes())) !=
        cudaSuccess)
        return cuda_fail(e, "tc_bwd_chunk_grads smem");
    launch_begin("tc_bwd_chunk_grads", st);
    // one CTA per SM walking the (chunk, head, batch) items
    const long long items = (long long)nc * (long long)H * (long long)bt;
    const unsigned pgrid = (unsigned)std::min<long long>(items, bwd_num_sms());
    tc_bwd_chunk_grads_kernel<<<pgrid, kThreads2, smemM_bytes(), st>>>(mX, mdY, mB, mC, mDX, mDB,
                                                                        mDC, am);
    launch_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tc_bwd_chunk_grads launch");
    return SSD_OK;
}

}  // namespace ssd
