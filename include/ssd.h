/*
 * libssd — the scalar-decay selective state-space layer (Mamba-2 "SSD") on
 * NVIDIA B200 (sm_100a). C ABI: plain pointers, sizes and status codes.
 *
 * The layer. For batch b, time t, head h (group g = h / (H/G)), head-dim p,
 * state index n:
 *
 *     h_t[p][n] = exp(dt_t * A_h) * h_{t-1}[p][n] + dt_t * x_t[p] * B_t[g][n]
 *     y_t[p]    = sum_n C_t[g][n] * h_t[p][n] + D_h * x_t[p]
 *
 * which equals the masked quadratic form y = (L o C B^T)(dt * X) with L the
 * 1-semiseparable decay mask L_ts = exp(dt_{s+1} A + ... + dt_t A), s <= t.
 * Sources: "Mamba-2 — 注意力的远亲" (docsaid.org), sections
 * "把 SSM 写成一个矩阵" (recurrence and matrix form M), "把 A 简化成一个数"
 * (scalar decay, M = L o (C B^T)), "跟着四个 token 算一次" (update the state,
 * then read it; the recurrent form serves generation) and "两条路各走一半"
 * (the chunked algorithm); "Mamba-2 模型解读", section 6.2 (the block
 * function takes initial states and returns Y and the final state); the decay
 * exp(Delta A) of "精读笔记 #12：Mamba", section 2.2.
 *
 * Conventions shared by every entry point:
 *   - Memory: all tensor pointers are DEVICE pointers, dense row-major
 *     (last index fastest), owned by the caller; the library never frees
 *     or keeps them. x, B, C, y, h, h0 and h_final must be 16-byte aligned;
 *     dt 2-byte (bf16) or 4-byte (fp32); A and D 4-byte.
 *   - Types: x, dt, B, C and y share one I/O type (ssd_dims.dtype: fp32 or
 *     bf16). A, D and every state (h0, h_final, h) are fp32. Accumulation
 *     and the carried state are fp32.
 *   - dt is the positive step AFTER any bias and softplus (ssd_forward_ex
 *     and ssd_step_ex take raw steps and prepare them, see ssd_options);
 *     A_h < 0 is the usual case (A_h >= 0 is computed as written and may
 *     overflow).
 *   - Limits: headdim P in {16, 32, ..., 128}; dstate N in {16, 32, ..., 256};
 *     nheads % ngroups == 0; batch >= 1; seqlen >= 0 (0 copies h0 to h_final).
 *   - Streams: every call only enqueues work on `stream` (NULL = the legacy
 *     default stream) and returns without synchronising.
 *   - Errors: arguments are validated before anything is enqueued; on any
 *     non-OK status nothing was enqueued unless the status is SSD_ERR_CUDA
 *     (a launch failed), and ssd_last_error() describes the failure.
 */
#ifndef LIBSSD_SSD_H
#define LIBSSD_SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSD_ABI_VERSION 2

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or workspace */
    SSD_ERR_UNSUPPORTED = 2, /* valid problem outside the supported limits */
    SSD_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed */
    SSD_ERR_NO_MEMORY = 4,   /* the library could not allocate workspace */
    SSD_ERR_TIMEOUT = 5      /* a device-side bounded wait gave up */
} ssd_status;

typedef enum ssd_dtype { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/* Problem sizes. `dtype` is the ssd_dtype of x, dt, B, C and y. */
typedef struct ssd_dims {
    int64_t batch;   /* b */
    int64_t seqlen;  /* L (ignored by ssd_step) */
    int64_t nheads;  /* H */
    int64_t headdim; /* P */
    int64_t dstate;  /* N */
    int64_t ngroups; /* G: B and C are shared by H/G consecutive heads */
    int32_t dtype;   /* ssd_dtype */
    int32_t reserved; /* must be 0 */
} ssd_dims;

/*
 * Step options of ssd_forward_ex and ssd_step_ex ("精读笔记 #12：Mamba",
 * llm-papers-study: section 3, algorithm 2 makes the step a softplus of a
 * projection; section 2.2 gives the zero-order hold rule
 * B_bar = (Delta A)^-1 (exp(Delta A) - I) Delta B). The dt argument then
 * holds RAW steps, prepared per element inside the kernels:
 *
 *     dt = raw + dt_bias[h]                     (dt_bias NULL: no bias)
 *     dt = softplus(dt) = log(1 + exp(dt))      (dt_softplus nonzero)
 *     dt = min(max(dt, dt_min), dt_max)         (only when dt_max > 0)
 *
 * The decay is always exp(dt * A_h). The input weight that multiplies
 * x_t (x) B_t is dt (SSD_DISC_EULER, the layer above) or, with
 * SSD_DISC_ZOH, (exp(dt * A_h) - 1) / A_h (dt where A_h = 0), the hold rule
 * for a scalar A. A zero-initialised struct means: no bias, no softplus, no
 * clamp, Euler weight, i.e. exactly ssd_forward / ssd_step.
 */
typedef enum ssd_discretization {
    SSD_DISC_EULER = 0,
    SSD_DISC_ZOH = 1
} ssd_discretization;

typedef struct ssd_options {
    const float *dt_bias;   /* (nheads) fp32 device array, 4-byte aligned, or NULL */
    int32_t dt_softplus;    /* nonzero: apply softplus after the bias */
    int32_t discretization; /* ssd_discretization */
    float dt_min;           /* clamp bounds: applied when dt_max > 0, then */
    float dt_max;           /*   0 <= dt_min <= dt_max is required */
    int32_t reserved[4];    /* must be 0 */
} ssd_options;

/* A CUDA stream; binary-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st *ssd_stream;

/*
 * Bytes of device workspace ssd_forward needs for these sizes and this
 * chunk length (0 when none). Returns 0 and sets ssd_last_error() for
 * invalid sizes as well; call ssd_forward to get the status.
 */
size_t ssd_forward_workspace_size(const ssd_dims *dims, int chunk);

/*
 * Prefill / training forward of the layer over whole sequences, by the
 * chunked state-space-duality algorithm ("两条路各走一半"; "Mamba-2 模型解读"
 * sections 6.1-6.2): within each block of `chunk` tokens the quadratic
 * (masked-attention) form; between blocks only the block-end state is passed.
 *
 *   x        (batch, seqlen, nheads, headdim)   I/O type
 *   dt       (batch, seqlen, nheads)            I/O type, > 0
 *   A        (nheads)                           fp32
 *   B, C     (batch, seqlen, ngroups, dstate)   I/O type
 *   D        (nheads) fp32, or NULL for no skip term
 *   h0       (batch, nheads, headdim, dstate) fp32 initial state, or NULL
 *            for zeros
 *   chunk    block length, one of 16, 32, 64, 128, 256. The result does not
 *            depend on it beyond rounding; it sets the work split.
 *   y        (batch, seqlen, nheads, headdim)   I/O type, written
 *   h_final  (batch, nheads, headdim, dstate) fp32, written, or NULL
 *   workspace, workspace_bytes
 *            device scratch of at least ssd_forward_workspace_size() bytes,
 *            256-byte aligned, or NULL: the library then allocates and frees
 *            it stream-ordered on `stream` (SSD_ERR_NO_MEMORY on failure).
 *            The workspace must not be shared by calls that may overlap.
 *   y may not alias any input; h_final may alias h0.
 *
 * Returns SSD_OK once all work is enqueued.
 */
ssd_status ssd_forward(const void *x, const void *dt, const float *A,
                       const void *B, const void *C, const float *D,
                       const float *h0, int chunk, void *y, float *h_final,
                       const ssd_dims *dims, void *workspace,
                       size_t workspace_bytes, ssd_stream stream);

/*
 * ssd_forward with step options (see ssd_options): dt holds raw steps,
 * prepared inside the kernels. opts NULL is ssd_forward. Invalid options
 * (a bad discretization, nonzero reserved words, dt_min < 0 or
 * dt_min > dt_max with dt_max > 0, a misaligned dt_bias) return
 * SSD_ERR_INVALID_ARG before anything is enqueued.
 */
ssd_status ssd_forward_ex(const void *x, const void *dt, const float *A,
                          const void *B, const void *C, const float *D,
                          const float *h0, int chunk, void *y, float *h_final,
                          const ssd_dims *dims, const ssd_options *opts,
                          void *workspace, size_t workspace_bytes,
                          ssd_stream stream);

/*
 * ssd_forward for callers that cannot allocate device memory. The pages
 * have no counterpart to this entry point; it is a deployment convenience.
 *
 * Some programs may not allocate on the device once they are running. A
 * serving process may have reserved all GPU memory for its own pool, so a
 * cudaMalloc would fail. A real-time loop may not allow an allocation's
 * latency or implicit synchronisation. A plain C caller may have no device
 * allocator at hand. This call takes the same arguments as ssd_forward minus
 * the workspace. Its scratch is a fixed 32 MiB array compiled into the
 * library. Every GPU that loads the library holds that array until the
 * process exits. The caller still provides every input and output.
 *
 *   - Nothing is allocated: no cudaMalloc/cudaFree and no allocating
 *     library call.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress while that device is current; make that first
 *     call before any stream capture. Later calls reuse the address. The
 *     address belongs to the device's primary context (the one the CUDA
 *     runtime uses): it does not survive cudaDeviceReset, and the entry
 *     point is not for contexts a caller creates through the driver API.
 *   - Problems whose workspace (ssd_forward_workspace_size) exceeds 32 MiB
 *     are rejected with SSD_ERR_UNSUPPORTED and a message giving both sizes.
 *   - All calls on a device share the one array, which keeps whatever the
 *     last call left in it. Each call writes every scratch word before it
 *     reads it, so no clearing is needed. Calls whose GPU work may overlap
 *     (different streams, or different host threads) race on it: serialise
 *     them, or use ssd_forward with separate workspaces.
 */
ssd_status ssd_forward_noalloc(const void *x, const void *dt, const float *A,
                               const void *B, const void *C, const float *D,
                               const float *h0, int chunk, void *y,
                               float *h_final, const ssd_dims *dims,
                               ssd_stream stream);

/*
 * One-token decode step, in place: the recurrent form the pages recommend
 * for generation ("跟着四个 token 算一次": the recurrence carries a fixed-size
 * state). One loop-body iteration of the definition above for every
 * (batch, head):
 *
 *   h   (batch, nheads, headdim, dstate) fp32, read and overwritten
 *   x   (batch, nheads, headdim)         I/O type
 *   dt  (batch, nheads)                  I/O type, > 0
 *   A   (nheads) fp32;  D (nheads) fp32 or NULL
 *   B, C (batch, ngroups, dstate)        I/O type
 *   y   (batch, nheads, headdim)         I/O type, written
 *
 * dims->seqlen is ignored. y may not alias h or any input.
 */
ssd_status ssd_step(float *h, const void *x, const void *dt, const float *A,
                    const void *B, const void *C, const float *D, void *y,
                    const ssd_dims *dims, ssd_stream stream);

/*
 * ssd_step with step options (see ssd_options): dt holds the raw step of
 * each (batch, head). opts NULL is ssd_step; invalid options as for
 * ssd_forward_ex.
 */
ssd_status ssd_step_ex(float *h, const void *x, const void *dt, const float *A,
                       const void *B, const void *C, const float *D, void *y,
                       const ssd_dims *dims, const ssd_options *opts,
                       ssd_stream stream);

/*
 * Sequence parallelism ("两条路各走一半": between blocks only the block-end
 * state passes; the same holds between consecutive pieces of a sequence held
 * by different GPUs). A sequence split into `nparts` consecutive pieces
 * (piece r on rank r) runs as:
 *   1. each rank: ssd_forward_state on its piece -> its end state S_r (from a
 *      zero initial state) and total decay Lambda_r = exp(sum_t dt_t A_h);
 *   2. an all-gather of (S_r, Lambda_r) across ranks (the caller's
 *      collective, e.g. NCCL);
 *   3. each rank: ssd_state_chain -> the state entering its piece,
 *      h_in = h0 chained through pieces 0..r-1 (h <- Lambda h + S);
 *   4. each rank: ssd_forward(_ex) on its piece with h0 = h_in.
 * The result equals the forward over the whole sequence up to rounding.
 */

/* Bytes of device workspace ssd_forward_state needs (0 when none). */
size_t ssd_forward_state_workspace_size(const ssd_dims *dims, int chunk);

/*
 * End state and total decay of each (batch, head) lane's sequence, from a
 * zero initial state, without computing y:
 *
 *   x (batch, seqlen, nheads, headdim), dt (batch, seqlen, nheads),
 *   B (batch, seqlen, ngroups, dstate)        I/O type, as for ssd_forward
 *   A (nheads) fp32; chunk as for ssd_forward
 *   state_out (batch, nheads, headdim, dstate) fp32, written, 16-byte aligned
 *   decay_out (batch, nheads) fp32, written: exp(sum_t dt_t A_h)
 *   opts     step options as for ssd_forward_ex (NULL: none)
 *   workspace, workspace_bytes as for ssd_forward (its own size function)
 *
 * seqlen 0 gives a zero state and decay 1.
 */
ssd_status ssd_forward_state(const void *x, const void *dt, const float *A,
                             const void *B, int chunk, float *state_out,
                             float *decay_out, const ssd_dims *dims,
                             const ssd_options *opts, void *workspace,
                             size_t workspace_bytes, ssd_stream stream);

/*
 * The state entering piece `part` (0 <= part < nparts) of a split sequence:
 *
 *   states (nparts, batch, nheads, headdim, dstate) fp32: the pieces' end
 *          states from ssd_forward_state, piece-major (the layout of an
 *          all-gather along the first axis)
 *   decays (nparts, batch, nheads) fp32: the pieces' total decays
 *   h0     (batch, nheads, headdim, dstate) fp32 state before piece 0, or
 *          NULL for zeros
 *   h_in   written (nullable): h0 chained through pieces 0 .. part-1
 *   h_total written (nullable): h0 chained through every piece, the whole
 *          sequence's final state
 *
 * dims gives batch, nheads, headdim, dstate (seqlen ignored). At least one
 * of h_in and h_total must be given; states, h0, h_in, h_total 16-byte
 * aligned.
 */
ssd_status ssd_state_chain(const float *states, const float *decays, int nparts,
                           int part, const float *h0, float *h_in, float *h_total,
                           const ssd_dims *dims, ssd_stream stream);

/*
 * The selective scan with a DIAGONAL A per channel ("精读笔记 #12：Mamba",
 * llm-papers-study, sections 2.2 and 3, algorithm 2), the recurrent layer the
 * SSD pages compare against. Every channel d carries its own N-vector state;
 * dims->nheads is the number of channels D and dims->headdim must be 1:
 *
 *   x, dt, y (batch, seqlen, D)        I/O type; dt as for ssd_forward(_ex)
 *   A        (D, dstate) fp32           the diagonal of each channel's A
 *   B, C     (batch, seqlen, ngroups, dstate) I/O type, shared by the D/G
 *            channels of a group; 4-element aligned
 *   Dskip    (D) fp32 or NULL;  h0, h_final (batch, D, dstate) fp32 or NULL
 *   opts     step options (bias per channel, softplus, clamp, Euler or
 *            zero-order-hold weight), NULL for none
 *
 *   h[n] = exp(dt A[d][n]) h[n] + w[n] x B[n],  y = sum_n C[n] h[n] + Dskip x
 *
 * with w[n] = dt (Euler) or (exp(dt A[d][n]) - 1) / A[d][n] (SSD_DISC_ZOH).
 * dstate must be 4, 8 or 16 (SSD_ERR_UNSUPPORTED otherwise).
 */
ssd_status ssd_selective_scan(const void *x, const void *dt, const float *A,
                              const void *B, const void *C, const float *Dskip,
                              const float *h0, void *y, float *h_final,
                              const ssd_dims *dims, const ssd_options *opts,
                              ssd_stream stream);

/*
 * Backward pass of the layer (the plain forward of ssd_forward: decay
 * exp(dt A_h), input weight dt; step options are not differentiated), by the
 * chunked decomposition with the chunk states recomputed ("精读笔记 #12：
 * Mamba", section 3.3: states are recomputed, not stored). bf16 I/O with
 * headdim 64 and dstate 128 runs its per-chunk products on the tensor cores
 * (128-token chunks, operands split into bf16 hi + lo pairs); every other size
 * runs on CUDA cores.
 * For the scalar loss sum dy . y + sum dh_final . h_final:
 *
 *   x, dt, A, B, C, D, h0   the forward's inputs (layouts of ssd_forward)
 *   dy       (batch, seqlen, nheads, headdim)  I/O type
 *   dh_final (batch, nheads, headdim, dstate) fp32 or NULL (zeros)
 *   dx (batch, seqlen, nheads, headdim), ddt (batch, seqlen, nheads),
 *   dA (nheads), dB, dC (batch, seqlen, ngroups, dstate), dD (nheads): fp32,
 *      written; dA and dD always required, the others when seqlen > 0 (dB,
 *      dC, dA, dD are summed over the heads and lanes that share them)
 *   dh0 (batch, nheads, headdim, dstate) fp32, written, or NULL
 *   workspace, workspace_bytes: as for ssd_forward, sized by
 *      ssd_backward_workspace_size
 *   x, B, C, dy, dx, dB, dC, h0, dh_final and dh0 must be 16-byte aligned
 *   (SSD_ERR_INVALID_ARG otherwise); dt, ddt, A, dA, D, dD to their types
 *
 * Sizes whose chunk tiles do not fit one CTA's shared memory return
 * SSD_ERR_UNSUPPORTED.
 */
size_t ssd_backward_workspace_size(const ssd_dims *dims);
ssd_status ssd_backward(const void *x, const void *dt, const float *A,
                        const void *B, const void *C, const float *D,
                        const float *h0, const void *dy, const float *dh_final,
                        float *dx, float *ddt, float *dA, float *dB, float *dC,
                        float *dD, float *dh0, const ssd_dims *dims,
                        void *workspace, size_t workspace_bytes,
                        ssd_stream stream);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word for the current device: SSD_OK, or SSD_ERR_TIMEOUT when a kernel's
 * bounded wait gave up since the last query, or SSD_ERR_CUDA when the
 * stream itself reports an error.
 */
ssd_status ssd_device_status(ssd_stream stream);

/* Message for the calling thread's most recent non-OK status ("" if none). */
const char *ssd_last_error(void);

/*
 * Test hook for the failure path (instrumentation, not part of the layer).
 * The tensor-core forward's pipelined warps, and the tensor-core backward's
 * kernels, wait on shared-memory barriers for their copies and tensor-core
 * work; every such wait is bounded, and a wait that runs out makes the kernel
 * stop its own work, let its copies and tensor-core operations in flight
 * finish, free its tensor memory, store nothing, and report SSD_ERR_TIMEOUT
 * through ssd_device_status. `cycles` is that bound in SM clock cycles for
 * kernels launched after the call, process-wide; 0 (or a negative value)
 * restores the default of about 2 s. A bound of a few cycles makes the next
 * forward or backward give up at its first wait that is not already
 * satisfied: its outputs are then undefined, and a later call with the
 * default bound computes normally.
 */
void ssd_set_wait_limit(long long cycles);

/*
 * Launch accounting and per-kernel timing (instrumentation, not part of the
 * layer). Every kernel the library launches is counted. Between
 * ssd_profile_begin() and ssd_profile_end() each launch is also bracketed by
 * two CUDA events recorded on the stream it was launched on.
 */
typedef struct ssd_kernel_time {
    const char *name;   /* static kernel name, owned by the library */
    long long launches; /* launches timed in the window */
    double total_ms;    /* sum of their event-measured durations */
} ssd_kernel_time;

/* Kernels launched by this library in this process so far. */
long long ssd_launch_count(void);

/* Opens a timing window (discarding any previous one). */
ssd_status ssd_profile_begin(void);

/*
 * Closes the window, waits for its events, and writes one entry per kernel
 * name into out[0 .. max_entries-1]. Returns the number of entries, or -1
 * (with ssd_last_error() set) if an event failed or the window overflowed
 * its 65536-launch capacity.
 */
int ssd_profile_end(ssd_kernel_time *out, int max_entries);

/* SSD_ABI_VERSION of the loaded library. */
int ssd_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBSSD_SSD_H */
