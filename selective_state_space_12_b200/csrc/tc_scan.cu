// Tensor-core forward path (sm_100a: TMA + tcgen05 + TMEM) for bf16 I/O,
// head dim P = 64, state N in {64, 128, 256}.
//
// The chunked algorithm ("Mamba-2 — 注意力的远亲", section "两条路各走一半";
// "Mamba-2 模型解读", sections 6.1-6.2) with blocks of 128 tokens: inside a
// block the quadratic (masked attention) form on tensor cores; between
// blocks only the block-end state passes on. One CTA walks the blocks of one
// (batch, head, segment) in order and carries the state on chip, so x is
// read once and y written once. Per 128-token block:
//
//   a0  cum_j = sum_{k<=j} dt_k A_h        (log2 units; decay warp)
//   a1  G  = C B^T                          tcgen05, TMEM fp32 [128 x 128]
//       Gm = G o L o dt + D I, L_ij = exp(cum_i - cum_j) for j <= i, else 0
//            (written back to TMEM as a bf16 hi + lo pair: A operands)
//       Yd = Gm_hi X + Gm_lo X              tcgen05, A from TMEM
//   a4  Yo = C H^T                          tcgen05 (H = state entering the block)
//       y  = Yd + exp(cum_i) Yo             epilogue, TMA store
//   a2  S^T = B^T (w o X), w_j = exp(cum_end - cum_j) dt_j   (w o X as bf16 hi + lo)
//   a3  H  <- exp(cum_end) H + S            fp32, in registers
//
// The skip term D x rides on the diagonal of Gm, so the epilogue needs no x.
// y leaves by bulk stores from shared memory (per-thread row stores, each
// warp instruction touching 32 rows, clog the load/store path that every
// shared-memory and mbarrier access of the CTA also takes). With two stages
// the epilogue writes y over the block's X tile, which then goes back to the
// producer once the store has read it; with one stage (N = 256) that would
// hold the next block's X behind the epilogue, so y goes through an 8 KB
// staging tile, 64 rows per store, and X is released as soon as the diagonal
// MMA and w o X have read it.
//
// Sequences with few (batch, head) lanes are cut into segments (about two
// waves of CTAs): a state-only
// pass gives each segment's local end state, the inter-chunk state pass
// (state_pass_launch) chains the segments, and the full pass starts each
// segment from its entering state. The state-only pass needs no recurrence: it
// walks a segment's blocks from the last to the first, weights token j by its
// decay to the end of the segment (exp2 of a non-positive exponent, the decay
// of the blocks already visited included), and accumulates every block's
// contribution in one TMEM accumulator, with w o X double-buffered so that
// the state group and the MMA overlap. With many lanes, those that would make a
// partial last wave of CTAs are cut in two instead: their first halves come
// first in the grid, every other lane whole after them, their second halves
// last; a second half starts from the state its first half left in global
// memory (a flag says it is there, long before the second half runs).
//
// Warp roles (512 threads). Warp group 0: warp 0 issues the TMA loads; warp 1
// issues the Gram, state->output (Yo) and diagonal MMAs; warp 2 issues the
// chunk-state MMAs, the only ones on the state recurrence; warp 3 computes
// each block's decay tables (cum, the weights w, the mask factors) up to four
// blocks ahead. Warp groups 1-3 (TMEM lane quarter = warp % 4): the state
// group (w o X, the state update), the mask group, the epilogue group. The
// state group forms block it's w o X as soon as block it-1's chunk state has
// been read, so the state update overlaps the next chunk-state MMA.
#include <cudaTypedefs.h>
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kBlk = 128;   // tokens per block
constexpr int kP = 64;      // head dim of this path
constexpr int kGroup = 128;                 // threads per math group (4 warps)
constexpr int kThreads = 4 * kGroup;
constexpr int kSlots = 3;                   // decay tables in flight
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at B200 clocks
constexpr float kLog2e = 1.4426950408889634f;
// The mask factor exp2(c_i - c_j) dt_j is formed as exp2(c_i - r) * (exp2(r - c_j) dt_j)
// with r the cum at the first token of j's 32-token group, when the cum falls
// by at most this much (log2 units) across the group: the second factor then
// stays below 2^96 dt_j, and a first factor that underflows stands for a true
// value below 2^-30 dt_j. Otherwise each element takes its own exp2.
constexpr float kSpanMax = 96.f;

enum { kFull = 0, kStateOnly = 1 };

// error codes written into the library's device error word
constexpr unsigned kErrWaitProducer = 0x101, kErrWaitMma = 0x102, kErrWaitState = 0x104,
                   kErrWaitMask = 0x108, kErrWaitEpi = 0x110, kErrWaitDecay = 0x120,
                   kErrWaitHalf = 0x140;

template <int N>
struct Cfg {
    static constexpr int kStages = (N <= 128) ? 2 : 1;
    static constexpr int kAtoms = N / 64;                   // 64-wide state slices
    static constexpr int kTile = kBlk * 128;                // one 128-row x 128-byte tile
    static constexpr int kXBytes = kTile;                   // X: 128 tokens x 64 bf16
    static constexpr int kCBytes = kAtoms * kTile;          // C: 128 tokens x N bf16
    // B: 128 tokens x N bf16; for N = 64 a second, all-zero atom follows it so
    // that B^T reads as a 128-row operand of the state MMA
    static constexpr int kBBytes = (N == 64 ? 2 : kAtoms) * kTile;
    static constexpr int kStageBytes = kXBytes + kBBytes + kCBytes;
    static constexpr int kHBytes = N * 128;                 // H^T bf16: N rows x 64
    static constexpr int oStage = 0;
    // w o X is rounded to bf16 as a pair hi + lo (both operands of the state
    // MMA), so the state keeps ~16 significant bits of each input term.
    static constexpr int oWX = oStage + kStages * kStageBytes;  // hi
    static constexpr int oWXlo = oWX + kTile;                   // lo
    static constexpr int oH = oWXlo + kTile;
    // state pass (no C tiles): the second w o X buffer lives in the C area,
    // hi in stage 0's C tile, lo after it or (N = 64) in stage 1's
    static constexpr int oC0 = oStage + kXBytes + kBBytes;
    static constexpr int oWX1 = oC0;
    static constexpr int oWX1lo = (kCBytes >= 2 * kTile) ? oC0 + kTile : oC0 + kStageBytes;
    // y staging (one stage only): 64 rows x 128 bytes
    static constexpr bool kYStage = (kStages == 1);
    static constexpr int oY = oH + kHBytes;
    static constexpr int oSmall = oY + (kYStage ? kTile / 2 : 0);
    static constexpr int kMB = (N >= 128) ? N / 128 : 1;    // state MMA M-blocks
    // With one M-block the chunk-state MMA takes w o X hi and lo side by side
    // as one 128-wide operand (two 64-column atoms 16 KB apart): S^T comes out
    // as 64 hi columns then 64 lo columns, summed by the state group. Wide
    // MMAs keep the tensor pipe far busier per instruction than 64-wide ones.
    static constexpr bool kMerged = (kMB == 1);
    // TMEM columns. Two Gram buffers (fp32); the mask group overwrites each
    // 32-column group in place with the masked Gram as bf16 hi (first 16
    // columns) and lo (last 16), the A operands of the diagonal MMA. Then Yd,
    // Yo, and the chunk state (128 columns).
    static constexpr uint32_t cG0 = 0, cG1 = 128, cYd = 256, cYo = 320, cS = 384;
};

// Decay tables of one block, written by the decay warp (token index within
// the block; c = cum in log2 units).
struct Tab {
    float c2[kBlk];   // c_i
    float w[kBlk];    // exp2(c_end - c_j) dt_j: weight of token j in the block-end state
    float v[kBlk];    // exp2(r_J - c_j) dt_j, r_J = c at the first token of j's group
                      // (dt_j in w and v: the input weight, as in `dt` below)
    float dt[kBlk];   // input weight of token j: dt_j or its zero-order hold (0 past the end)
    float r[4];       // r_J
    int sep[4];       // group J takes the two-factor form
    float d;          // exp2(c_end): decay of the state across the block
    float pad[3];
};

struct Small {
    Tab tab[kSlots];
    int abort;
    uint32_t tmem_base;
    uint64_t full_x[2], empty_x[2];   // TMA stage: X tile filled / free
    uint64_t full_bc[2], empty_bc[2]; // TMA stage: B and C tiles filled / free
    uint64_t tab_full[kSlots], tab_free[kSlots];  // decay tables written / read by all
    uint64_t gram_full[2], gm_full[2]; // per Gram buffer: Gram done / masked
    uint64_t wx_full, state_full, h_full, hbf_free, out_full, y_free, drain;
    uint64_t wxb_full[2], wxb_free[2];  // state pass: w o X buffer filled / read by the MMA
    float prep[2][kBlk];  // step options: the decay warp's prepared dt and input weight
};

static_assert(offsetof(Small, prep) % 16 == 0, "prep is read as float4");

// dynamic shared memory of one CTA: the tiles, the small state, alignment slack
template <int N>
constexpr int smem_bytes() {
    return Cfg<N>::oSmall + ((int)sizeof(Small) + 127) / 128 * 128 + 1024;
}
static_assert(smem_bytes<64>() <= 227 * 1024 && smem_bytes<128>() <= 227 * 1024 &&
                  smem_bytes<256>() <= 227 * 1024,
              "shared memory");

struct ScanArgs {
    const __nv_bfloat16 *dt;
    const float *A;
    const float *D;
    const float *h_init;  // state entering each CTA's first block (layout per lane [p][n]) or NULL
    float *h_out;         // final state (full pass, one segment) / local end state (state pass)
    float *seg_decay;     // state pass: exp(sum of dt*A over the segment)
    unsigned int *err;
    // clock cycles a pipeline wait may take before the CTA gives up (the
    // drains that follow an abort keep kWaitCycles)
    long long wait;
    int L, H, G, nb, nseg;
    int h_init_stride_seg;  // 1 when h_init is per segment (workspace), 0 when per lane (h0)
    // lanes cut in two (the last n_cut lanes; 1-D grid: first halves, whole
    // lanes, second halves); blocks [0, cut_blk) and [cut_blk, nb)
    int n_cut, cut_blk;
    float *half_state;       // per cut lane: the state after its first half
    unsigned int *half_flag; // per cut lane: set once that state is out
    DtPreArgs pre;           // step options (kernels instantiated with PRE only)
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    // byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Bounded wait that gives up once the CTA has aborted. A math thread that
// gives up keeps executing the same sequence of named barriers as the rest of
// its group (so no barrier is left short); its results are discarded and
// nothing is stored. Every mbarrier access is a shared-memory round trip: the
// phase is tested first, then waited for in hardware (the thread sleeps until
// the phase completes or the suspend hint runs out), and the abort flag is
// read only between sleeps. The slow path is out of line so that the hot code
// stays small (the instruction cache serves sixteen warps in six roles).
template <bool HINT>
__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, int *abort,
                                       unsigned int *err, long long limit, unsigned code) {
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait<HINT>(bar, parity)) return true;
        if (*(volatile int *)abort) return false;
        if (clock64() - t0 > limit) {
            *(volatile int *)abort = 1;
            atomicOr(err, code);
            return false;
        }
    }
}

template <bool HINT>
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, int *abort,
                                              unsigned int *err, long long limit, unsigned code) {
    if (mbar_test_wait(bar, parity)) return true;
    return wait_slow<HINT>(bar, parity, abort, err, limit, code);
}

// Waits for two phases; both are tested at once first, so that when both have
// completed the caller pays one round trip.
template <bool HINT>
__device__ __noinline__ bool wait2_slow(uint64_t *b1, uint32_t p1, uint64_t *b2, uint32_t p2,
                                        int *abort, unsigned int *err, long long limit,
                                        unsigned code) {
    return wait_or_abort<HINT>(b1, p1, abort, err, limit, code) &&
           wait_or_abort<HINT>(b2, p2, abort, err, limit, code);
}
template <bool HINT>
__device__ __forceinline__ bool wait2_or_abort(uint64_t *b1, uint32_t p1, uint64_t *b2, uint32_t p2,
                                               int *abort, unsigned int *err, long long limit,
                                               unsigned code) {
    const bool t1 = mbar_test_wait(b1, p1);
    const bool t2 = mbar_test_wait(b2, p2);
    if (t1 && t2) return true;
    return wait2_slow<HINT>(b1, p1, b2, p2, abort, err, limit, code);
}

// The same for three phases.
template <bool HINT>
__device__ __noinline__ bool wait3_slow(uint64_t *b1, uint32_t p1, uint64_t *b2, uint32_t p2,
                                        uint64_t *b3, uint32_t p3, int *abort, unsigned int *err,
                                        long long limit, unsigned code) {
    return wait_or_abort<HINT>(b1, p1, abort, err, limit, code) &&
           wait_or_abort<HINT>(b2, p2, abort, err, limit, code) &&
           wait_or_abort<HINT>(b3, p3, abort, err, limit, code);
}
template <bool HINT>
__device__ __forceinline__ bool wait3_or_abort(uint64_t *b1, uint32_t p1, uint64_t *b2, uint32_t p2,
                                               uint64_t *b3, uint32_t p3, int *abort,
                                               unsigned int *err, long long limit, unsigned code) {
    const bool t1 = mbar_test_wait(b1, p1);
    const bool t2 = mbar_test_wait(b2, p2);
    const bool t3 = mbar_test_wait(b3, p3);
    if (t1 && t2 && t3) return true;
    return wait3_slow<HINT>(b1, p1, b2, p2, b3, p3, abort, err, limit, code);
}


// Per-row factors of the mask for the 32-column groups J = 0..3 of one block:
// u_J = exp2(c_i - r_J) and whether group J takes the two-factor form. Read
// from the decay tables before the Gram is ready.
struct RowMask {
    float u[4];
    bool sep[4];
};

__device__ __forceinline__ RowMask row_mask(const Tab &T, float c2i) {
    RowMask m;
    const float4 r = *reinterpret_cast<const float4 *>(T.r);
    const int4 sp = *reinterpret_cast<const int4 *>(T.sep);
    m.u[0] = fast_exp2(c2i - r.x);
    m.u[1] = fast_exp2(c2i - r.y);
    m.u[2] = fast_exp2(c2i - r.z);
    m.u[3] = fast_exp2(c2i - r.w);
    m.sep[0] = sp.x != 0;
    m.sep[1] = sp.y != 0;
    m.sep[2] = sp.z != 0;
    m.sep[3] = sp.w != 0;
    return m;
}

// Decay-mask the Gram row held by this thread (row i = `row`, lane quarter
// q), in place, group by group: each 32-column group's fp32 values become 16
// bf16x2 columns of the masked value's hi part and 16 of its lo part. Groups
// J < q lie wholly below the diagonal; group q holds the diagonal (columns
// j > i are zero, and D is added at j = i); groups J > q are zero.
__device__ __forceinline__ void mask_row(uint32_t gaddr, int q, int row, float c2i, float Dh,
                                         const Tab &T, const RowMask &m) {
#pragma unroll 1
    for (int J = 0; J <= q; ++J) {
        const float u = J == 0 ? m.u[0] : J == 1 ? m.u[1] : J == 2 ? m.u[2] : m.u[3];
        const bool sep = J == 0 ? m.sep[0] : J == 1 ? m.sep[1] : J == 2 ? m.sep[2] : m.sep[3];
        uint32_t gr[32];
        tmem_ld32(gaddr + 32 * J, gr);
        float g[32];
        if (sep) {
            // factor u * v_j (v read before the TMEM wait)
            float4 vv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) vv[k] = *reinterpret_cast<const float4 *>(T.v + 32 * J + 4 * k);
            tmem_wait_ld();
            reg_fence32(gr);
            const f2 u2 = f2_pack(u, u);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                f2_unpack(f2_mul(f2_mul(f2_pack(__uint_as_float(gr[4 * k]), __uint_as_float(gr[4 * k + 1])),
                                        f2_pack(vv[k].x, vv[k].y)), u2), g[4 * k], g[4 * k + 1]);
                f2_unpack(f2_mul(f2_mul(f2_pack(__uint_as_float(gr[4 * k + 2]), __uint_as_float(gr[4 * k + 3])),
                                        f2_pack(vv[k].z, vv[k].w)), u2), g[4 * k + 2], g[4 * k + 3]);
            }
        } else {
            // decay span too wide for the two-factor form: one exp2 per element
            tmem_wait_ld();
            reg_fence32(gr);
#pragma unroll
            for (int k = 0; k < 32; ++k)
                g[k] = __uint_as_float(gr[k]) * (fast_exp2(c2i - T.c2[32 * J + k]) * T.dt[32 * J + k]);
        }
        if (J == q) {
            // the diagonal group (column 32 q + k against row 32 q + l): zero
            // above the diagonal, D on it
            const int l = row & 31;
#pragma unroll
            for (int k = 0; k < 32; ++k) g[k] = (k < l) ? g[k] : ((k == l) ? g[k] + Dh : 0.f);
        }
        uint32_t pk[16], pl[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) split_bf16x2(g[2 * k], g[2 * k + 1], pk[k], pl[k]);
        tmem_st16(gaddr + 32 * J, pk);
        tmem_st16(gaddr + 32 * J + 16, pl);
    }
}

// (a2) Row `row` of w o X as bf16 hi + lo (the X tile's swizzled layout), in
// packed bf16x2 arithmetic: w = w_hi + w_lo; hi = w_hi x rounded; the exact
// residual w_hi x - hi by one fused multiply-add; lo = w_lo x + residual. Two
// 16-byte chunks per trip: the loads of a trip go out before their uses; the
// loop stays rolled to keep the hot code small.
__device__ __forceinline__ void form_wx(const unsigned char *xt, float wj, unsigned char *dhi,
                                        unsigned char *dlo, int row) {
    const uint32_t wh = pack_bf16(wj, wj);
    const float whf = bf16_lo(wh);
    const uint32_t wl = pack_bf16(wj - whf, wj - whf);
    constexpr int kPass = 2;
#pragma unroll 1
    for (int c0 = 0; c0 < 8; c0 += kPass) {
        uint4 xv[kPass];
#pragma unroll
        for (int c = 0; c < kPass; ++c)
            xv[c] = *reinterpret_cast<const uint4 *>(xt + swz(row, c0 + c));
#pragma unroll
        for (int c = 0; c < kPass; ++c) {
            const uint32_t xw[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                hw[u] = mul_bf16x2(wh, xw[u]);
                const uint32_t res = fma_bf16x2(wh, xw[u], hw[u] ^ 0x80008000u);
                lw[u] = fma_bf16x2(wl, xw[u], res);
            }
            const uint32_t off = swz(row, c0 + c);
            *reinterpret_cast<uint4 *>(dhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(dlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
}

// PRE: dt holds raw steps, prepared per token by the decay warp (bias,
// softplus, clamp; zero-order-hold input weight); without it, the kernel
// reads prepared steps and the input weight is dt itself.
template <int N, int MODE, bool PRE>
__global__ void __launch_bounds__(kThreads, 1)
tc_scan_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
               const ScanArgs a) {
    using K = Cfg<N>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned base, derived from the __shared__ array by an offset so
    // that the compiler keeps shared-space loads and stores (not generic ones)
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Small *sm = reinterpret_cast<Small *>(smem + K::oSmall);

    // this CTA's lane and blocks; part 1 / 2: first / second half of a cut lane
    int seg, h, b, blk0, blk1, part = 0, cut = 0;
    if (a.n_cut > 0) {
        const int lanes = (int)(gridDim.x) - a.n_cut, c = (int)blockIdx.x;
        int bh;
        if (c < a.n_cut) {
            part = 1;
            cut = c;
            bh = lanes - a.n_cut + c;
            blk0 = 0;
            blk1 = a.cut_blk;
        } else if (c < lanes) {
            bh = c - a.n_cut;
            blk0 = 0;
            blk1 = a.nb;
        } else {
            part = 2;
            cut = c - lanes;
            bh = lanes - a.n_cut + cut;
            blk0 = a.cut_blk;
            blk1 = a.nb;
        }
        seg = 0;
        b = bh / a.H;
        h = bh - b * a.H;
    } else {
        seg = blockIdx.x;
        h = blockIdx.y;
        b = blockIdx.z;
        blk0 = (int)((long long)seg * a.nb / a.nseg);
        blk1 = (int)((long long)(seg + 1) * a.nb / a.nseg);
    }
    const int g = h / (a.H / a.G);
    const int nit = blk1 - blk0;
    // block of trip `it`: in order on the full pass, last to first on the state pass
    const int blk_step = MODE == kStateOnly ? -1 : 1;
    const int blk_first = MODE == kStateOnly ? blk1 - 1 : blk0;
    auto blk_of = [=](int it) { return blk_first + blk_step * it; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wg = warp >> 2;  // warp group

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm->full_x[s], 1);
            // full pass: the diagonal MMA and the state group (y staged apart),
            // or the epilogue once y, written over the tile, has been stored;
            // state pass: the state group
            mbar_init(&sm->empty_x[s], (MODE == kFull && K::kYStage) ? 2 : 1);
            mbar_init(&sm->full_bc[s], 1);
            mbar_init(&sm->empty_bc[s], MODE == kFull ? 2 : 1);  // one per MMA issuer
            mbar_init(&sm->gram_full[s], 1);
            mbar_init(&sm->gm_full[s], 1);
        }
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sm->tab_full[s], 1);
            mbar_init(&sm->tab_free[s], MODE == kFull ? 3 : 1);  // state, mask, epilogue groups
        }
        mbar_init(&sm->wx_full, 1);
        mbar_init(&sm->state_full, 1);
        mbar_init(&sm->h_full, 1);
        mbar_init(&sm->hbf_free, 1);
        mbar_init(&sm->out_full, 2);  // diagonal MMA + Yo MMA
        mbar_init(&sm->y_free, 1);
        mbar_init(&sm->drain, MODE == kFull ? 2 : 1);
        if (MODE == kStateOnly) {
            for (int s = 0; s < 2; ++s) {
                mbar_init(&sm->wxb_full[s], 1);
                mbar_init(&sm->wxb_free[s], 1);
            }
        }
        sm->abort = 0;
        fence_mbar_init();
    }
    if (N == 64) {  // the zero atom after each stage's B tile (never loaded by TMA)
        for (int s = 0; s < K::kStages; ++s) {
            uint4 *z = reinterpret_cast<uint4 *>(smem + K::oStage + s * K::kStageBytes +
                                                 K::kXBytes + K::kTile);
            for (int i = threadIdx.x; i < K::kTile / 16; i += blockDim.x)
                z[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&sm->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (wg == 0) {
        if (warp == 0 && lane == 0) {
            // -------------------------------------------- TMA producer
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmB);
            if (MODE == kFull) {
                tma_prefetch_desc(&tmC);
                tma_prefetch_desc(&tmY);
            }
            const uint32_t bc_bytes = (MODE == kFull ? 2 : 1) * K::kAtoms * K::kTile;
            // the tiles of block `it` pulled into L2 a few blocks ahead of their loads
            constexpr int kAhead = 3;
            auto prefetch = [&](int it) {
                const int t0 = blk_of(it) * kBlk;
                tma_prefetch_l2_4d(&tmX, 0, h, t0, b);
                for (int q = 0; q < K::kAtoms; ++q) {
                    tma_prefetch_l2_4d(&tmB, 64 * q, g, t0, b);
                    if (MODE == kFull) tma_prefetch_l2_4d(&tmC, 64 * q, g, t0, b);
                }
            };
            for (int it = 1; it < kAhead && it < nit; ++it) prefetch(it);
            int issued_bc = 0, issued_x = 0;
            for (int it = 0; it < nit; ++it) {
                const int s = it % K::kStages;
                const int r = it / K::kStages;  // refill number of stage s
                if (it + kAhead < nit) prefetch(it + kAhead);
                unsigned char *st = smem + K::oStage + s * K::kStageBytes;
                const int t0 = blk_of(it) * kBlk;
                if (r > 0 && !wait_or_abort<PRE>(&sm->empty_bc[s], (r - 1) & 1, &sm->abort, a.err, a.wait,
                                            kErrWaitProducer))
                    break;
                mbar_arrive_expect_tx(&sm->full_bc[s], bc_bytes);
                for (int q = 0; q < K::kAtoms; ++q) {
                    tma_load_4d(st + K::kXBytes + q * K::kTile, &tmB, &sm->full_bc[s], 64 * q, g,
                                t0, b);
                    if (MODE == kFull)
                        tma_load_4d(st + K::kXBytes + K::kBBytes + q * K::kTile, &tmC,
                                    &sm->full_bc[s], 64 * q, g, t0, b);
                }
                ++issued_bc;
                if (r > 0 && !wait_or_abort<PRE>(&sm->empty_x[s], (r - 1) & 1, &sm->abort, a.err, a.wait,
                                            kErrWaitProducer))
                    break;
                mbar_arrive_expect_tx(&sm->full_x[s], K::kXBytes);
                tma_load_4d(st, &tmX, &sm->full_x[s], 0, h, t0, b);
                ++issued_x;
            }
            // on an abort, let the loads already issued land before the CTA exits
            if (*(volatile int *)&sm->abort) {
                for (int it = (issued_bc > K::kStages ? issued_bc - K::kStages : 0);
                     it < issued_bc; ++it)
                    mbar_wait(&sm->full_bc[it % K::kStages], (it / K::kStages) & 1, kWaitCycles);
                for (int it = (issued_x > K::kStages ? issued_x - K::kStages : 0); it < issued_x;
                     ++it)
                    mbar_wait(&sm->full_x[it % K::kStages], (it / K::kStages) & 1, kWaitCycles);
            }
        } else if ((warp == 1 || warp == 2) && lane == 0) {
            // -------------------------------------------- MMA issuers
            // Two threads on different SM sub-partitions issue independent
            // chains: warp 1 the Gram and diagonal MMAs (block it+1's Gram goes
            // out before block it's diagonal MMA waits for its mask), warp 2 the
            // chunk-state MMA of block it and then its Yo, so that the state
            // recurrence never waits behind the output side. Descriptors are
            // built once per operand and advanced by constant offsets (start
            // address field = address / 16).
            constexpr uint32_t iGram = idesc_bf16(128, 128, false, false);
            constexpr uint32_t iOff = idesc_bf16(128, 64, false, true);
            constexpr uint32_t iState = idesc_bf16(128, 64, true, true);
            constexpr uint32_t iDiag = idesc_bf16(128, 64, false, true);
            const uint32_t base = smem_u32(smem);
            int *ab = &sm->abort;
            auto stage_addr = [&](int it) {
                return base + K::oStage + (it % K::kStages) * K::kStageBytes;
            };
            const bool out_issuer = (warp == 1);
            if (out_issuer && MODE == kFull) {
                // G = C B^T into Gram buffer it & 1: both K-major, K = state dim
                auto gram = [&](int it) -> bool {
                    if (!wait_or_abort<PRE>(&sm->full_bc[it % K::kStages], (it / K::kStages) & 1, ab,
                                       a.err, a.wait, kErrWaitMma))
                        return false;
                    tc_fence_after();
                    const uint32_t st = stage_addr(it);
                    const uint64_t dc = sdesc_sw128(st + K::kXBytes + K::kBBytes, 16, 1024);
                    const uint64_t db = sdesc_sw128(st + K::kXBytes, 16, 1024);
                    const uint32_t dg = tmem + ((it & 1) ? K::cG1 : K::cG0);
#pragma unroll
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t off = ((k >> 2) * K::kTile + (k & 3) * 32) >> 4;
                        mma_ss(dg, dc + off, db + off, iGram, k > 0);
                    }
                    mma_commit(&sm->gram_full[it & 1]);
                    mma_commit(&sm->empty_bc[it % K::kStages]);
                    return true;
                };
                bool ok = nit > 0 ? gram(0) : true;
                for (int it = 0; it < nit && ok; ++it) {
                    const int s = it % K::kStages;
                    // with two stages block it+1's B and C are already on their
                    // way; with one they come after this block's Yo
                    if (K::kStages > 1 && it + 1 < nit && !gram(it + 1)) break;
                    // Yd = Gm X with Gm (bf16 hi + lo, in place in Gram buffer it & 1),
                    // once the epilogue group has read block it-1's Yd (before
                    // block 0, y_free's phase "-1" counts as complete)
                    if (!wait3_or_abort<PRE>(&sm->gm_full[it & 1], (it >> 1) & 1, &sm->full_x[s],
                                        (it / K::kStages) & 1, &sm->y_free, (it - 1) & 1, ab, a.err, a.wait,
                                        kErrWaitMma))
                        break;
                    tc_fence_after();
                    {
                        const uint32_t ag = tmem + ((it & 1) ? K::cG1 : K::cG0);
                        const uint64_t dx = sdesc_sw128(stage_addr(it), 1024, 1024);
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)  // 16 tokens: 8 columns of a 32-col group
                            mma_ts(tmem + K::cYd, ag + 32 * (k >> 1) + 8 * (k & 1),
                                   dx + (k * 2048 >> 4), iDiag, k > 0);
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)
                            mma_ts(tmem + K::cYd, ag + 32 * (k >> 1) + 16 + 8 * (k & 1),
                                   dx + (k * 2048 >> 4), iDiag, 1);
                    }
                    mma_commit(&sm->out_full);
                    if (K::kYStage) mma_commit(&sm->empty_x[s]);
                    if (K::kStages == 1 && it + 1 < nit && !gram(it + 1)) break;
                }
                mma_commit(&sm->drain);
                mbar_wait(&sm->drain, 0, kWaitCycles);
            } else if (!out_issuer && MODE == kStateOnly) {
                // state pass: every block's contribution into one accumulator,
                // w o X from two buffers (block parity)
                constexpr uint32_t iState2 = idesc_bf16(128, 128, true, true);
                for (int it = 0; it < nit; ++it) {
                    const int s = it % K::kStages, wb = it & 1;
                    const uint32_t st = stage_addr(it);
                    if (!wait2_or_abort<PRE>(&sm->full_bc[s], (it / K::kStages) & 1, &sm->wxb_full[wb],
                                        (it >> 1) & 1, ab, a.err, a.wait, kErrWaitMma))
                        break;
                    tc_fence_after();
                    const uint32_t hi = base + (wb ? K::oWX1 : K::oWX);
                    const uint32_t lo = base + (wb ? K::oWX1lo : K::oWXlo);
                    const uint64_t dbt = sdesc_sw128(st + K::kXBytes, K::kTile, 1024);
                    if (K::kMB == 1) {
                        const uint64_t dw = sdesc_sw128(hi, lo - hi, 1024);  // hi | lo
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)
                            mma_ss(tmem + K::cS, dbt + (k * 2048 >> 4), dw + (k * 2048 >> 4), iState2,
                                   it > 0 || k > 0);
                    } else {
                        const uint64_t dh = sdesc_sw128(hi, 1024, 1024);
                        const uint64_t dl = sdesc_sw128(lo, 1024, 1024);
#pragma unroll
                        for (int m = 0; m < K::kMB; ++m) {
#pragma unroll
                            for (int k = 0; k < kBlk / 16; ++k)
                                mma_ss(tmem + K::cS + 64 * m,
                                       dbt + ((2 * m * K::kTile + k * 2048) >> 4),
                                       dh + (k * 2048 >> 4), iState, it > 0 || k > 0);
#pragma unroll
                            for (int k = 0; k < kBlk / 16; ++k)
                                mma_ss(tmem + K::cS + 64 * m,
                                       dbt + ((2 * m * K::kTile + k * 2048) >> 4),
                                       dl + (k * 2048 >> 4), iState, 1);
                        }
                    }
                    mma_commit(&sm->wxb_free[wb]);
                    mma_commit(&sm->empty_bc[s]);
                }
                mma_commit(&sm->state_full);
                mma_commit(&sm->drain);
                mbar_wait(&sm->drain, 0, kWaitCycles);
            } else if (!out_issuer) {
                constexpr uint32_t iState2 = idesc_bf16(128, 128, true, true);
                const uint64_t dwx = sdesc_sw128(base + K::oWX, 1024, 1024);
                const uint64_t dwxlo = sdesc_sw128(base + K::oWXlo, 1024, 1024);
                const uint64_t dwx2 = sdesc_sw128(base + K::oWX, K::kTile, 1024);  // hi | lo
                const uint64_t dh = sdesc_sw128(base + K::oH, 1024, 1024);
                for (int it = 0; it < nit; ++it) {
                    const int s = it % K::kStages;
                    const uint32_t st = stage_addr(it);
                    // S^T = B^T (w o X): A = B tile read M-major (state contiguous).
                    // wx_full also says that the state group has read S of block it-1.
                    if (!wait2_or_abort<PRE>(&sm->full_bc[s], (it / K::kStages) & 1, &sm->wx_full, it & 1,
                                        ab, a.err, a.wait, kErrWaitMma))
                        break;
                    tc_fence_after();
                    const uint64_t dbt = sdesc_sw128(st + K::kXBytes, K::kTile, 1024);
                    if (K::kMerged) {
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)
                            mma_ss(tmem + K::cS, dbt + (k * 2048 >> 4), dwx2 + (k * 2048 >> 4),
                                   iState2, k > 0);
                    } else {
#pragma unroll
                    for (int m = 0; m < K::kMB; ++m) {
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)
                            mma_ss(tmem + K::cS + 64 * m, dbt + ((2 * m * K::kTile + k * 2048) >> 4),
                                   dwx + (k * 2048 >> 4), iState, k > 0);
#pragma unroll
                        for (int k = 0; k < kBlk / 16; ++k)
                            mma_ss(tmem + K::cS + 64 * m, dbt + ((2 * m * K::kTile + k * 2048) >> 4),
                                   dwxlo + (k * 2048 >> 4), iState, 1);
                    }
                    }
                    mma_commit(&sm->state_full);
                    if (MODE == kFull) {
                        // Yo = C H^T (H = state entering this block), once the
                        // epilogue group has read block it-1's Yo
                        if (!wait2_or_abort<PRE>(&sm->h_full, it & 1, &sm->y_free, (it - 1) & 1, ab,
                                            a.err, a.wait, kErrWaitMma))
                            break;
                        tc_fence_after();
                        const uint32_t dyo = tmem + K::cYo;
                        const uint64_t dc = sdesc_sw128(st + K::kXBytes + K::kBBytes, 16, 1024);
#pragma unroll
                        for (int k = 0; k < N / 16; ++k) {
                            const uint32_t off = ((k >> 2) * K::kTile + (k & 3) * 32) >> 4;
                            mma_ss(dyo, dc + off, dh + (k * 2048 >> 4), iOff, k > 0);
                        }
                        mma_commit(&sm->hbf_free);
                        mma_commit(&sm->out_full);
                    }
                    mma_commit(&sm->empty_bc[s]);  // B and C are read by no later MMA
                }
                mma_commit(&sm->drain);
                mbar_wait(&sm->drain, 0, kWaitCycles);
            }
        } else if (warp == 3) {
            // -------------------------------------------- decay warp
            // lane holds tokens 4 lane .. 4 lane + 3 of each block
            const float Araw = a.A[h];
            const float Ah = Araw * kLog2e;
            const float pre_bias = (PRE && a.pre.bias) ? a.pre.bias[h] : 0.f;
            const float inv_A = (PRE && Araw != 0.f) ? 1.f / Araw : 0.f;
            int *ab = &sm->abort;
            // lane holds tokens 4 lane + k; with PRE, the raw steps of tokens
            // 32 k + lane instead (one token per lane per preparation pass)
            auto load_dt = [&](int blk, float (&d)[4]) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int t = blk * kBlk + (PRE ? 32 * k + lane : 4 * lane + k);
                    d[k] = (t < a.L) ? __bfloat162float(a.dt[((long long)b * a.L + t) * a.H + h])
                                     : 0.f;
                }
            };
            float dtn[4] = {0.f, 0.f, 0.f, 0.f};
            if (nit > 0) load_dt(blk_of(0), dtn);
            float seg_total2 = 0.f;
            for (int it = 0; it < nit; ++it) {
                const int slot = it % kSlots;
                float dv[4], c[4], in4[4];
                if (PRE) {
                    // the block's raw steps, prepared one token per lane per pass
                    // (rolled, so that the math appears once in the hot code):
                    // dt for the decay, the input weight for w, v and the table
                    float r = dtn[0];
#pragma unroll 1
                    for (int k = 0; k < 4; ++k) {
                        const int j = 32 * k + lane;
                        const bool live = blk_of(it) * kBlk + j < a.L;  // else no decay, no input
                        const float d = live ? prepare_dt_compact(r, pre_bias, a.pre) : 0.f;
                        sm->prep[0][j] = d;
                        sm->prep[1][j] = input_weight_compact(d, Araw, inv_A, a.pre.zoh);
                        r = k == 0 ? dtn[1] : k == 1 ? dtn[2] : dtn[3];
                    }
                    __syncwarp();
                    const float4 d4 = *reinterpret_cast<const float4 *>(&sm->prep[0][4 * lane]);
                    const float4 w4v = *reinterpret_cast<const float4 *>(&sm->prep[1][4 * lane]);
                    dv[0] = d4.x; dv[1] = d4.y; dv[2] = d4.z; dv[3] = d4.w;
                    in4[0] = w4v.x; in4[1] = w4v.y; in4[2] = w4v.z; in4[3] = w4v.w;
                    __syncwarp();
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) dv[k] = in4[k] = dtn[k];
                }
                if (it + 1 < nit) load_dt(blk_of(it + 1), dtn);
                // (a0) cum within the block: 4 tokens per lane, then across the warp
                float run = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    run += dv[k] * Ah;
                    c[k] = run;
                }
                float incl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += u;
                }
                const float excl = incl - run;
#pragma unroll
                for (int k = 0; k < 4; ++k) c[k] += excl;
                const float total2 = __shfl_sync(0xffffffffu, incl, 31);
                const int g0 = lane & ~7;  // first lane of this lane's 32-token group
                const float rJ = __shfl_sync(0xffffffffu, c[0], g0);
                const float endJ = __shfl_sync(0xffffffffu, c[3], g0 + 7);
                if (it >= kSlots)
                    wait_or_abort<PRE>(&sm->tab_free[slot], ((it - kSlots) / kSlots) & 1, ab, a.err, a.wait,
                                  kErrWaitDecay);
                Tab &T = sm->tab[slot];
                float w4[4], v4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // (in4: the input weight, dt or its zero-order hold)
                    // state pass: decay to the end of the segment; seg_total2 holds
                    // the blocks already visited (the later ones)
                    w4[k] = fast_exp2((MODE == kStateOnly ? seg_total2 + total2 : total2) - c[k]) *
                            in4[k];
                    v4[k] = fast_exp2(rJ - c[k]) * in4[k];
                }
                *reinterpret_cast<float4 *>(T.c2 + 4 * lane) = make_float4(c[0], c[1], c[2], c[3]);
                *reinterpret_cast<float4 *>(T.w + 4 * lane) = make_float4(w4[0], w4[1], w4[2], w4[3]);
                *reinterpret_cast<float4 *>(T.v + 4 * lane) = make_float4(v4[0], v4[1], v4[2], v4[3]);
                *reinterpret_cast<float4 *>(T.dt + 4 * lane) = make_float4(in4[0], in4[1], in4[2], in4[3]);
                if (lane == g0) {
                    T.r[lane >> 3] = rJ;
                    T.sep[lane >> 3] = (fabsf(rJ - endJ) <= kSpanMax) ? 1 : 0;
                }
                if (lane == 0) T.d = fast_exp2(total2);
                seg_total2 += total2;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->tab_full[slot]);
            }
            if (MODE == kStateOnly && lane == 0 && !*(volatile int *)ab) {
                const long long lane_bh = (long long)b * a.H + h;
                a.seg_decay[lane_bh * a.nseg + seg] = exp2f(seg_total2);
            }
        }
    } else if (wg == 1 && MODE == kStateOnly) {
        // ------------------------------------------------ state group, state pass
        // block by block (last to first) w o X into the buffer of the block's
        // parity; the chunk-state MMA accumulates all of them
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const bool leader = (q == 0 && lane == 0);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const long long lane_bh = (long long)b * a.H + h;
        int *ab = &sm->abort;
        for (int it = 0; it < nit; ++it) {
            const int s = it % K::kStages, wb = it & 1;
            wait2_or_abort<PRE>(&sm->tab_full[it % kSlots], (it / kSlots) & 1, &sm->full_x[s],
                           (it / K::kStages) & 1, ab, a.err, a.wait, kErrWaitState);
            if (it >= 2) wait_or_abort<PRE>(&sm->wxb_free[wb], ((it - 2) >> 1) & 1, ab, a.err, a.wait, kErrWaitState);
            const float wj = sm->tab[it % kSlots].w[row];
            form_wx(smem + K::oStage + s * K::kStageBytes, wj, smem + (wb ? K::oWX1 : K::oWX),
                    smem + (wb ? K::oWX1lo : K::oWXlo), row);
            fence_proxy_async_smem();
            named_bar(1, kGroup);
            if (leader) {
                mbar_arrive(&sm->wxb_full[wb]);
                mbar_arrive(&sm->empty_x[s]);
                mbar_arrive(&sm->tab_free[it % kSlots]);
            }
        }
        // the segment's local end state: the accumulator (hi + lo columns for N <= 128)
        wait_or_abort<PRE>(&sm->state_full, 0, ab, a.err, a.wait, kErrWaitState);
        tc_fence_after();
        float *ho = a.h_out + (lane_bh * a.nseg + seg) * (long long)kP * N;
        const bool ok = !*(volatile int *)ab;
#pragma unroll
        for (int m = 0; m < K::kMB; ++m) {
            const int n = row + 128 * m;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[32];
                tmem_ld32(tmem + lane_base + K::cS + 64 * m + 32 * half, sv);
                tmem_wait_ld();
                reg_fence32(sv);
                float v[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(sv[k]);
                if (K::kMB == 1) {  // lo columns follow the hi ones
                    tmem_ld32(tmem + lane_base + K::cS + 64 + 32 * half, sv);
                    tmem_wait_ld();
                    reg_fence32(sv);
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] += __uint_as_float(sv[k]);
                }
                if (ok && n < N) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) ho[(long long)(32 * half + k) * N + n] = v[k];
                }
            }
        }
    } else if (wg == 1) {
        // ------------------------------------------------ state group
        // thread owns token `row` (w o X) and state rows row + 128 m. Trip it
        // takes block it-1's chunk state into H, forms block it's w o X, then
        // publishes H (the state entering block it) for block it's Yo.
        const int q = warp & 3;          // TMEM lane quarter
        const int row = 32 * q + lane;
        const bool leader = (q == 0 && lane == 0);
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const long long lane_bh = (long long)b * a.H + h;
        unsigned char *wxp = smem + K::oWX;
        unsigned char *wxlp = smem + K::oWXlo;
        unsigned char *hbp = smem + K::oH;
        int *ab = &sm->abort;

        float H[K::kMB][64];
        {
            const float *hi = nullptr;
            if (MODE == kFull && part == 2) {
                // the second half of a cut lane: wait (bounded) for the first
                // half's state, written early in the kernel by another CTA
                if (leader) {
                    const long long t0 = clock64();
                    while (ld_acquire_u32(&a.half_flag[cut]) == 0u) {
                        if (*(volatile int *)ab) break;
                        if (clock64() - t0 > a.wait) {
                            *(volatile int *)ab = 1;
                            atomicOr(a.err, kErrWaitHalf);
                            break;
                        }
                        __nanosleep(512);
                    }
                }
                named_bar(1, kGroup);
                hi = a.half_state + (long long)cut * kP * N;
            } else if (MODE == kFull && a.h_init) {
                hi = a.h_init + (lane_bh * (a.h_init_stride_seg ? a.nseg : 1) +
                                 (a.h_init_stride_seg ? seg : 0)) *
                                    (long long)kP * N;
            }
#pragma unroll
            for (int m = 0; m < K::kMB; ++m) {
                const int n = row + 128 * m;
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    H[m][k] = (hi && n < N) ? __ldcg(hi + (long long)k * N + n) : 0.f;
            }
        }
        auto write_hbf = [&]() {
#pragma unroll
            for (int m = 0; m < K::kMB; ++m) {
                const int n = row + 128 * m;
                if (n >= N) continue;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v;
                    v.x = pack_bf16(H[m][8 * c + 0], H[m][8 * c + 1]);
                    v.y = pack_bf16(H[m][8 * c + 2], H[m][8 * c + 3]);
                    v.z = pack_bf16(H[m][8 * c + 4], H[m][8 * c + 5]);
                    v.w = pack_bf16(H[m][8 * c + 6], H[m][8 * c + 7]);
                    *reinterpret_cast<uint4 *>(hbp + swz(n, c)) = v;
                }
            }
        };
        if (MODE == kFull) {
            write_hbf();
            fence_proxy_async_smem();
            named_bar(1, kGroup);
            if (leader) mbar_arrive(&sm->h_full);
        }
        for (int it = 0; it <= nit; ++it) {
            const int s = it % K::kStages;
            // With two stages, block it's tables and X tile, and the factors d
            // (block it-1) and w (block it), are fetched before the wait for
            // block it-1's chunk state, so that their round trips overlap that
            // MMA. (With one stage, block it's X arrives only after block it-1's
            // MMAs, so the state update goes first.)
            float d = 0.f, wj = 0.f;
            auto fetch = [&]() {
                if (it < nit)
                    wait2_or_abort<PRE>(&sm->tab_full[it % kSlots], (it / kSlots) & 1,
                                   &sm->full_x[s], (it / K::kStages) & 1, ab, a.err, a.wait, kErrWaitState);
                if (it > 0) d = sm->tab[(it - 1) % kSlots].d;
                if (it < nit) wj = sm->tab[it % kSlots].w[row];
            };
            if (K::kStages > 1) fetch();
            if (K::kStages == 1 && it > 0) d = sm->tab[(it - 1) % kSlots].d;
            if (it > 0) {
                // (a3) H <- exp(cum_end) H + S of block it-1
                wait_or_abort<PRE>(&sm->state_full, (it - 1) & 1, ab, a.err, a.wait, kErrWaitState);
                tc_fence_after();
                if (K::kMerged) {
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {  // 16 state columns: hi + lo
                        uint32_t sh[16], sl[16];
                        tmem_ld16(tmem + lane_base + K::cS + 16 * qq, sh);
                        tmem_ld16(tmem + lane_base + K::cS + 64 + 16 * qq, sl);
                        tmem_wait_ld();
                        reg_fence16(sh);
                        reg_fence16(sl);
                        const f2 d2 = f2_pack(d, d);
#pragma unroll
                        for (int k = 0; k < 16; k += 2) {
                            const f2 s2 = f2_add(f2_pack(__uint_as_float(sh[k]), __uint_as_float(sh[k + 1])),
                                                 f2_pack(__uint_as_float(sl[k]), __uint_as_float(sl[k + 1])));
                            f2_unpack(f2_fma(d2, f2_pack(H[0][16 * qq + k], H[0][16 * qq + k + 1]), s2),
                                      H[0][16 * qq + k], H[0][16 * qq + k + 1]);
                        }
                    }
                } else {
#pragma unroll
                for (int m = 0; m < K::kMB; ++m) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t sv[32];
                        tmem_ld32(tmem + lane_base + K::cS + 64 * m + 32 * half, sv);
                        tmem_wait_ld();
                        reg_fence32(sv);
                        const f2 d2 = f2_pack(d, d);
#pragma unroll
                        for (int k = 0; k < 32; k += 2)
                            f2_unpack(f2_fma(d2, f2_pack(H[m][32 * half + k], H[m][32 * half + k + 1]),
                                             f2_pack(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1]))),
                                      H[m][32 * half + k], H[m][32 * half + k + 1]);
                    }
                }
                }
            }
            if (K::kStages == 1) fetch();
            if (it < nit) {
                // (a2) w o X -> bf16 hi + lo (same swizzled layout as X), in packed
                // bf16x2 arithmetic: w = w_hi + w_lo; hi = w_hi x rounded; the exact
                // residual w_hi x - hi by one fused multiply-add; lo = w_lo x + residual
                const unsigned char *xt = smem + K::oStage + s * K::kStageBytes;
                const uint32_t wh = pack_bf16(wj, wj);
                const float whf = bf16_lo(wh);
                const uint32_t wl = pack_bf16(wj - whf, wj - whf);
                // two 16-byte chunks per trip: the loads of a trip go out before
                // their uses; the loop stays rolled to keep the hot code small
                constexpr int kPass = 2;
#pragma unroll 1
                for (int c0 = 0; c0 < 8; c0 += kPass) {
                    uint4 xv[kPass];
#pragma unroll
                    for (int c = 0; c < kPass; ++c)
                        xv[c] = *reinterpret_cast<const uint4 *>(xt + swz(row, c0 + c));
#pragma unroll
                    for (int c = 0; c < kPass; ++c) {
                        const uint32_t xw[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            hw[u] = mul_bf16x2(wh, xw[u]);
                            const uint32_t res = fma_bf16x2(wh, xw[u], hw[u] ^ 0x80008000u);
                            lw[u] = fma_bf16x2(wl, xw[u], res);
                        }
                        const uint32_t off = swz(row, c0 + c);
                        *reinterpret_cast<uint4 *>(wxp + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        *reinterpret_cast<uint4 *>(wxlp + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            named_bar(1, kGroup);
            if (leader) {
                if (it < nit) {
                    mbar_arrive(&sm->wx_full);
                    if (MODE == kStateOnly || K::kYStage) mbar_arrive(&sm->empty_x[s]);
                }
                if (it > 0) mbar_arrive(&sm->tab_free[(it - 1) % kSlots]);
            }
            if (MODE == kFull && it > 0 && it < nit) {
                // publish H for block it's Yo once block it-1's Yo has read the old one
                wait_or_abort<PRE>(&sm->hbf_free, (it - 1) & 1, ab, a.err, a.wait, kErrWaitState);
                write_hbf();
                fence_proxy_async_smem();
                named_bar(1, kGroup);
                if (leader) mbar_arrive(&sm->h_full);
            }
        }

        // final / local end state; the first half of a cut lane hands its state on
        if (!*(volatile int *)ab) {
            float *ho = nullptr;
            if (MODE == kFull && a.h_out) ho = a.h_out + lane_bh * (long long)kP * N;
            if (MODE == kFull && part == 1) ho = a.half_state + (long long)cut * kP * N;
            if (MODE == kStateOnly)
                ho = a.h_out + (lane_bh * a.nseg + seg) * (long long)kP * N;
            if (ho) {
#pragma unroll
                for (int m = 0; m < K::kMB; ++m) {
                    const int n = row + 128 * m;
                    if (n >= N) continue;
#pragma unroll
                    for (int k = 0; k < 64; ++k) ho[(long long)k * N + n] = H[m][k];
                }
            }
        }
        if (MODE == kFull && part == 1) {
            // all of the state is out before the flag goes up
            __threadfence();
            named_bar(1, kGroup);
            if (leader && !*(volatile int *)ab) st_release_u32(&a.half_flag[cut], 1u);
        }
    } else if (wg == 2) {
        // ------------------------------------------------ mask group
        if (MODE == kFull) {
            const int q = warp & 3;
            const int row = 32 * q + lane;
            const bool leader = (q == 0 && lane == 0);
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            const float Dh = a.D ? a.D[h] : 0.f;
            int *ab = &sm->abort;
            for (int it = 0; it < nit; ++it) {
                const int bb = it & 1;
                const int slot = it % kSlots;
                const uint32_t gbase = tmem + lane_base + (bb ? K::cG1 : K::cG0);
                wait_or_abort<PRE>(&sm->tab_full[slot], (it / kSlots) & 1, ab, a.err, a.wait, kErrWaitMask);
                const Tab &T = sm->tab[slot];
                const float c2i = T.c2[row];
                const RowMask rm = row_mask(T, c2i);
                // (a1) Gm = G o L o dt + D I for row i = row
                wait_or_abort<PRE>(&sm->gram_full[bb], (it >> 1) & 1, ab, a.err, a.wait, kErrWaitMask);
                tc_fence_after();
                mask_row(gbase, q, row, c2i, Dh, T, rm);
                {
                    uint32_t zero[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) zero[k] = 0u;
#pragma unroll 1
                    for (int J = q + 1; J < 4; ++J) {
                        tmem_st16(gbase + 32 * J, zero);
                        tmem_st16(gbase + 32 * J + 16, zero);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                named_bar(2, kGroup);
                if (leader) {
                    mbar_arrive(&sm->gm_full[bb]);
                    mbar_arrive(&sm->tab_free[slot]);
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue group
        if (MODE == kFull) {
            const int q = warp & 3;
            const int row = 32 * q + lane;
            const bool leader = (q == 0 && lane == 0);
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            int *ab = &sm->abort;
            for (int it = 0; it < nit; ++it) {
                const int slot = it % kSlots;
                // (a4) y = Yd + exp(cum_i) Yo; Yd and Yo are released as soon as
                // both halves are in registers
                wait2_or_abort<PRE>(&sm->tab_full[slot], (it / kSlots) & 1, &sm->out_full, it & 1, ab,
                               a.err, a.wait, kErrWaitEpi);
                const float e = fast_exp2(sm->tab[slot].c2[row]);
                const f2 e2 = f2_pack(e, e);
                tc_fence_after();
                uint32_t ow[32];
                {
                    uint32_t yd[32], yo[32];
                    tmem_ld32(tmem + lane_base + K::cYd, yd);
                    tmem_ld32(tmem + lane_base + K::cYo, yo);
                    tmem_wait_ld();
                    reg_fence32(yd);
                    reg_fence32(yo);
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float o0, o1;
                        f2_unpack(f2_fma(e2, f2_pack(__uint_as_float(yo[2 * k]), __uint_as_float(yo[2 * k + 1])),
                                         f2_pack(__uint_as_float(yd[2 * k]), __uint_as_float(yd[2 * k + 1]))),
                                  o0, o1);
                        ow[k] = pack_bf16(o0, o1);
                    }
                    tmem_ld32(tmem + lane_base + K::cYd + 32, yd);
                    tmem_ld32(tmem + lane_base + K::cYo + 32, yo);
                    tmem_wait_ld();
                    reg_fence32(yd);
                    reg_fence32(yo);
                    tc_fence_before();
                    named_bar(3, kGroup);
                    if (leader) {
                        mbar_arrive(&sm->y_free);
                        mbar_arrive(&sm->tab_free[slot]);
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float o0, o1;
                        f2_unpack(f2_fma(e2, f2_pack(__uint_as_float(yo[2 * k]), __uint_as_float(yo[2 * k + 1])),
                                         f2_pack(__uint_as_float(yd[2 * k]), __uint_as_float(yd[2 * k + 1]))),
                                  o0, o1);
                        ow[16 + k] = pack_bf16(o0, o1);
                    }
                }
                const int t0 = blk_of(it) * kBlk;
                if (K::kYStage) {
                    // y through the 8 KB staging tile: rows 0-63 (warps 0, 1), then
                    // rows 64-127 (warps 2, 3), one bulk store each
                    unsigned char *yst = smem + K::oY;
#pragma unroll 1
                    for (int hb = 0; hb < 2; ++hb) {
                        if ((q >> 1) == hb) {
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4 *>(yst + swz(row - 64 * hb, c)) = make_uint4(
                                    ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
                            fence_proxy_async_smem();
                        }
                        named_bar(3, kGroup);
                        if (leader && !*(volatile int *)ab && t0 + 64 * hb < a.L) {
                            tma_store_4d(&tmY, yst, 0, h, t0 + 64 * hb, b);
                            bulk_commit();
                            bulk_wait_read0();
                        }
                        named_bar(3, kGroup);  // the staging tile is free again
                    }
                } else {
                    // y over this block's X tile (dead: its MMAs and w o X are
                    // done), then one bulk store; the tile goes back to the
                    // producer once the store has read it
                    unsigned char *xt = smem + K::oStage + (it % K::kStages) * K::kStageBytes;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(xt + swz(row, c)) =
                            make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
                    fence_proxy_async_smem();
                    named_bar(3, kGroup);
                    if (leader) {
                        if (!*(volatile int *)ab) {
                            tma_store_4d(&tmY, xt, 0, h, t0, b);
                            bulk_commit();
                            bulk_wait_read0();
                        }
                        mbar_arrive(&sm->empty_x[it % K::kStages]);
                    }
                }
            }
            if (leader) bulk_wait0();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

ssd_status get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    return SSD_OK;
}

// 4-D bf16 map over a (d3, d2, d1, d0) row-major tensor, box {64, 1, rows, 1},
// 128-byte swizzle, zero fill outside the tensor.
ssd_status make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t d3, uint32_t rows = kBlk) {
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {64, 1, rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SSD_OK;
}

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int N, int MODE, bool PRE>
cudaError_t launch_scan(dim3 grid, const CUtensorMap &mx, const CUtensorMap &mb,
                        const CUtensorMap &mc, const CUtensorMap &my, const ScanArgs &args,
                        cudaStream_t st) {
    const int smem = smem_bytes<N>();
    cudaError_t e = cudaFuncSetAttribute(tc_scan_kernel<N, MODE, PRE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    launch_begin(MODE == kFull ? "tc_chunk_scan" : "tc_segment_state", st);
    tc_scan_kernel<N, MODE, PRE><<<grid, kThreads, smem, st>>>(mx, mb, mc, my, args);
    launch_end(st);
    return cudaGetLastError();
}

template <int MODE, bool PRE>
cudaError_t launch_np(int N, dim3 grid, const CUtensorMap &mx, const CUtensorMap &mb,
                      const CUtensorMap &mc, const CUtensorMap &my, const ScanArgs &args,
                      cudaStream_t st) {
    switch (N) {
        case 64: return launch_scan<64, MODE, PRE>(grid, mx, mb, mc, my, args, st);
        case 128: return launch_scan<128, MODE, PRE>(grid, mx, mb, mc, my, args, st);
        default: return launch_scan<256, MODE, PRE>(grid, mx, mb, mc, my, args, st);
    }
}

template <int MODE>
cudaError_t launch_n(int N, bool pre, dim3 grid, const CUtensorMap &mx, const CUtensorMap &mb,
                     const CUtensorMap &mc, const CUtensorMap &my, const ScanArgs &args,
                     cudaStream_t st) {
    return pre ? launch_np<MODE, true>(N, grid, mx, mb, mc, my, args, st)
               : launch_np<MODE, false>(N, grid, mx, mb, mc, my, args, st);
}

}  // namespace

bool tc_supported(const Problem &pr) {
    return pr.dtype == SSD_BF16 && pr.headdim == kP &&
           (pr.dstate == 64 || pr.dstate == 128 || pr.dstate == 256) &&
           (pr.chunk == 128 || pr.chunk == 256) && pr.seqlen > 0;
}

// Segments per (batch, head) lane: one when there are enough lanes to fill
// the GPU, else enough to give about two waves of CTAs (on the long sequence,
// 32 lanes on 148 SMs, one wave of segments took 469 us, two 444, three 476,
// four 486: longer segments pay their fill and drain less often, but a
// single wave leaves SMs idle).
int tc_segments(const Problem &pr) {
    const long long lanes = pr.batch * pr.nheads;
    const long long nb = (pr.seqlen + kBlk - 1) / kBlk;
    const long long sms = num_sms();
    if (lanes >= 2 * sms || nb < 4) return 1;
    long long nseg = (2 * sms) / lanes;
    nseg = nseg < 1 ? 1 : nseg;
    nseg = nseg > nb / 2 ? nb / 2 : nseg;
    return (int)(nseg < 1 ? 1 : nseg);
}

// With one segment per lane: the lanes past the last full wave of CTAs are
// cut in two when they are at most half a wave (so that their second halves
// find idle SMs when the whole lanes end) and hold at least two blocks.
int tc_cut_lanes(const Problem &pr) {
    if (tc_segments(pr) > 1) return 0;
    const long long lanes = pr.batch * pr.nheads;
    const long long nb = (pr.seqlen + kBlk - 1) / kBlk;
    const long long sms = num_sms();
    const long long cut = lanes % sms;
    if (lanes < sms || nb < 2 || cut == 0 || 2 * cut > sms) return 0;
    return (int)cut;
}

size_t tc_workspace_bytes(const Problem &pr) {
    const int nseg = tc_segments(pr);
    const int n_cut = tc_cut_lanes(pr);
    if (n_cut > 0)
        return align256((size_t)n_cut * kP * pr.dstate * 4) + align256((size_t)n_cut * 4);
    if (nseg <= 1) return 0;
    const size_t lanes = (size_t)(pr.batch * pr.nheads);
    return align256(lanes * nseg * (size_t)kP * pr.dstate * 4) + align256(lanes * nseg * 4);
}

size_t tc_state_workspace_bytes(const Problem &pr) {
    const int nseg = tc_segments(pr);
    if (nseg <= 1) return 0;
    const size_t lanes = (size_t)(pr.batch * pr.nheads);
    return align256(lanes * nseg * (size_t)kP * pr.dstate * 4) + align256(lanes * nseg * 4);
}

// The state-only pass alone: each segment's local end state and decay, then
// (several segments) the state pass from a zero state, which leaves the
// lane's end state and the product of the segment decays.
ssd_status tc_state(const Problem &pr, const void *x, const void *dt, const float *A,
                    const void *B, float *state_out, float *decay_out, void *ws, cudaStream_t st,
                    const DtPre &pre) {
    ssd_status s = get_encoder();
    if (s != SSD_OK) return s;
    const int N = (int)pr.dstate;
    CUtensorMap mx, mb;
    if ((s = make_map(&mx, x, kP, pr.nheads, pr.seqlen, pr.batch)) != SSD_OK) return s;
    if ((s = make_map(&mb, B, N, pr.ngroups, pr.seqlen, pr.batch)) != SSD_OK) return s;
    unsigned int *err = device_error_word();
    if (!err) return fail(SSD_ERR_CUDA, "cannot locate the device error word");
    const int nb = (int)((pr.seqlen + kBlk - 1) / kBlk);
    const int nseg = tc_segments(pr);
    const size_t lanes = (size_t)(pr.batch * pr.nheads);
    ScanArgs sa{};
    sa.dt = static_cast<const __nv_bfloat16 *>(dt);
    sa.A = A;
    sa.err = err;
    sa.wait = wait_limit_cycles();
    sa.L = (int)pr.seqlen;
    sa.H = (int)pr.nheads;
    sa.G = (int)pr.ngroups;
    sa.nb = nb;
    sa.nseg = nseg;
    sa.pre = DtPreArgs{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    float *seg_states = state_out, *seg_decay = decay_out;
    if (nseg > 1) {
        seg_states = static_cast<float *>(ws);
        seg_decay = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                              align256(lanes * nseg * (size_t)kP * N * 4));
    }
    sa.h_out = seg_states;
    sa.seg_decay = seg_decay;
    dim3 grid((unsigned)nseg, (unsigned)pr.nheads, (unsigned)pr.batch);
    cudaError_t e;
    // the state-only pass reads no C and writes no y: X's map stands in for both
    if ((e = launch_n<kStateOnly>(N, pre.active(), grid, mx, mb, mx, mx, sa, st)) != cudaSuccess)
        return cuda_fail(e, "tc_segment_state launch");
    if (nseg > 1)
        return state_pass_launch(seg_states, seg_decay, nullptr, state_out, pr.batch, pr.nheads,
                                 kP * N / 4, nseg, st, decay_out);
    return SSD_OK;
}

ssd_status tc_forward(const Problem &pr, const void *x, const void *dt, const float *A,
                      const void *B, const void *C, const float *D, const float *h0, void *y,
                      float *h_final, void *ws, cudaStream_t st, const DtPre &pre) {
    ssd_status s = get_encoder();
    if (s != SSD_OK) return s;
    const int N = (int)pr.dstate;
    CUtensorMap mx, my, mb, mc;
    if ((s = make_map(&mx, x, kP, pr.nheads, pr.seqlen, pr.batch)) != SSD_OK) return s;
    // y is stored 64 rows at a time with one stage (N = 256), a whole block otherwise
    if ((s = make_map(&my, y, kP, pr.nheads, pr.seqlen, pr.batch, N == 256 ? kBlk / 2 : kBlk)) !=
        SSD_OK)
        return s;
    if ((s = make_map(&mb, B, N, pr.ngroups, pr.seqlen, pr.batch)) != SSD_OK) return s;
    if ((s = make_map(&mc, C, N, pr.ngroups, pr.seqlen, pr.batch)) != SSD_OK) return s;
    unsigned int *err = device_error_word();
    if (!err) return fail(SSD_ERR_CUDA, "cannot locate the device error word");

    const int nb = (int)((pr.seqlen + kBlk - 1) / kBlk);
    const int nseg = tc_segments(pr);
    ScanArgs args{};
    args.dt = static_cast<const __nv_bfloat16 *>(dt);
    args.A = A;
    args.D = D;
    args.err = err;
    args.wait = wait_limit_cycles();
    args.L = (int)pr.seqlen;
    args.H = (int)pr.nheads;
    args.G = (int)pr.ngroups;
    args.nb = nb;
    args.nseg = nseg;
    args.pre = DtPreArgs{pre.bias, pre.softplus, pre.zoh, pre.dt_min, pre.dt_max};
    const bool pre_on = pre.active();
    dim3 grid((unsigned)nseg, (unsigned)pr.nheads, (unsigned)pr.batch);
    args.n_cut = 0;
    cudaError_t e;
    if (nseg > 1) {
        const size_t lanes = (size_t)(pr.batch * pr.nheads);
        float *seg_states = static_cast<float *>(ws);
        float *seg_decay = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                                     align256(lanes * nseg * (size_t)kP * N * 4));
        ScanArgs sa = args;
        sa.h_init = nullptr;
        sa.h_out = seg_states;
        sa.seg_decay = seg_decay;
        if ((e = launch_n<kStateOnly>(N, pre_on, grid, mx, mb, mc, my, sa, st)) != cudaSuccess)
            return cuda_fail(e, "tc_segment_state launch");
        if ((s = state_pass_launch(seg_states, seg_decay, h0, h_final, pr.batch, pr.nheads,
                                   kP * N / 4, nseg, st)) != SSD_OK)
            return s;
        args.h_init = seg_states;
        args.h_init_stride_seg = 1;
        args.h_out = nullptr;
    } else {
        args.h_init = h0;
        args.h_init_stride_seg = 0;
        args.h_out = h_final;
        const int n_cut = tc_cut_lanes(pr);
        if (n_cut > 0) {
            args.n_cut = n_cut;
            args.cut_blk = nb / 2;
            args.half_state = static_cast<float *>(ws);
            args.half_flag = reinterpret_cast<unsigned int *>(
                static_cast<char *>(ws) + align256((size_t)n_cut * kP * N * 4));
            if ((e = cudaMemsetAsync(args.half_flag, 0, (size_t)n_cut * 4, st)) != cudaSuccess)
                return cuda_fail(e, "half-lane flag reset");
            grid = dim3((unsigned)(pr.batch * pr.nheads + n_cut));
        }
    }
    if ((e = launch_n<kFull>(N, pre_on, grid, mx, mb, mc, my, args, st)) != cudaSuccess)
        return cuda_fail(e, "tc_chunk_scan launch");
    return SSD_OK;
}

}  // namespace ssd
