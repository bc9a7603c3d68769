// Host-side declarations shared by the libssd translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

struct Problem {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
    int dtype;  // ssd_dtype
    int chunk;
    int64_t nchunks() const { return chunk > 0 ? (seqlen + chunk - 1) / chunk : 0; }
};

// Step options as the kernels take them (ssd_options, validated): raw step
// -> + bias[h] -> softplus -> clamp when dt_max > 0; input weight dt or the
// zero-order hold (exp(dt A) - 1) / A.
struct DtPre {
    const float *bias = nullptr;
    int softplus = 0, zoh = 0;
    float dt_min = 0.f, dt_max = 0.f;
    bool active() const { return bias || softplus || zoh || dt_max > 0.f; }
};

// Records a message for ssd_last_error() and returns `s`.
ssd_status fail(ssd_status s, const char *fmt, ...);
ssd_status cuda_fail(cudaError_t e, const char *what);

// Rounds up to a multiple of 256 bytes.
inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// --- general (CUDA-core) forward path: any supported size, fp32 or bf16 ---
size_t simt_workspace_bytes(const Problem &pr);
ssd_status simt_forward(const Problem &pr, const void *x, const void *dt, const float *A,
                        const void *B, const void *C, const float *D, const float *h0,
                        void *y, float *h_final, void *ws, cudaStream_t st,
                        const DtPre &pre = DtPre());

// End state (from a zero initial state) and total decay of each lane's
// sequence, by the CUDA-core chunk states and state pass; workspace as for
// simt_forward.
ssd_status simt_state(const Problem &pr, const void *x, const void *dt, const float *A,
                      const void *B, float *state_out, float *decay_out, void *ws,
                      cudaStream_t st, const DtPre &pre = DtPre());

// Inter-chunk state pass over `nc` consecutive pieces per (batch, head) lane:
// S (lanes, nc, P*N) holds each piece's own end state on entry and the state
// entering each piece on exit; h_final (nullable) receives the final state and
// decay_total (nullable) the product of the pieces' decays.
ssd_status state_pass_launch(float *S, const float *decay, const float *h0, float *h_final,
                             int64_t batch, int64_t nheads, int PN4, int nc, cudaStream_t st,
                             float *decay_total = nullptr);

// Per-chunk states S (lanes, nc, P*N) and decays (lanes, nc) of the plain
// layer (chunk pr.chunk), or with `adjoint` the chunks' contributions
// sum_i exp(cum_i) dy_i (x) C_i to their entering state's gradient (x := dy,
// B := C).
ssd_status chunk_states_launch(const Problem &pr, const void *x, const void *dt, const float *A,
                               const void *B, float *S, float *decay, bool adjoint,
                               cudaStream_t st);

// Backward pass of the plain layer (CUDA cores), see backward.cu.
size_t backward_workspace_bytes(const Problem &pr);
int backward_chunk(const Problem &pr);  // 0: unsupported sizes
ssd_status backward_launch(const Problem &pr, const void *x, const void *dt, const float *A,
                           const void *B, const void *C, const float *D, const float *h0,
                           const void *dy, const float *dh_final, float *dx, float *ddt,
                           float *dA, float *dB, float *dC, float *dD, float *dh0, void *ws,
                           cudaStream_t st);

// Tensor-core per-chunk gradients (bf16 I/O, P = 64, N = 128, 128-token
// chunks), see tc_backward.cu. dB and dC must be zeroed: every head adds its
// share.
bool tc_backward_supported(const Problem &pr);
ssd_status tc_chunk_states(const Problem &pr, const void *x, const void *dt, const float *A,
                           const void *B, float *S, float *decay, bool adjoint, cudaStream_t st);
// The chunk states chained along each lane in one pass: the state entering
// each chunk (init = h0), or with adjoint the gradient at each chunk's end
// (init = dh_final) and final_out = dh0.
ssd_status tc_state_chain(const Problem &pr, const void *x, const void *dt, const float *A,
                          const void *B, const float *init, float *out, float *final_out,
                          bool adjoint, cudaStream_t st);
// Whether the problem has enough lanes for the chains to fill the GPU.
bool tc_chain_pays(const Problem &pr);
ssd_status tc_backward_chunks(const Problem &pr, const void *x, const void *dt, const float *A,
                              const void *B, const void *C, const float *D, const void *dy,
                              const float *Hst, const float *R, float *dx, float *ddt, float *dB,
                              float *dC, float *dA_part, float *dD_part, cudaStream_t st);

// Sequence parallelism: the state entering piece `part` of `nparts` from the
// pieces' end states S (nparts, lanes, P*N) and decays (nparts, lanes);
// h_total (nullable) receives the chain over all pieces.
ssd_status state_chain_launch(const float *S, const float *decays, const float *h0, float *h_in,
                              float *h_total, int64_t batch, int64_t nheads, int PN4, int nparts,
                              int part, cudaStream_t st);

// --- tensor-core forward path (bf16, P = 64, N in {64,128,256}, chunk 128/256) ---
bool tc_supported(const Problem &pr);
int tc_segments(const Problem &pr);
size_t tc_workspace_bytes(const Problem &pr);
ssd_status tc_forward(const Problem &pr, const void *x, const void *dt, const float *A,
                      const void *B, const void *C, const float *D, const float *h0, void *y,
                      float *h_final, void *ws, cudaStream_t st, const DtPre &pre = DtPre());
// End state and total decay by the state-only tensor-core pass (segments and
// the state pass when lanes are few); workspace tc_state_workspace_bytes.
size_t tc_state_workspace_bytes(const Problem &pr);
ssd_status tc_state(const Problem &pr, const void *x, const void *dt, const float *A,
                    const void *B, float *state_out, float *decay_out, void *ws, cudaStream_t st,
                    const DtPre &pre = DtPre());

// --- selective scan (diagonal A per channel; nheads = channels, headdim 1) ---
bool scan_supported_dstate(int64_t N);
ssd_status scan_launch(const Problem &pr, const void *x, const void *dt, const float *A,
                       const void *B, const void *C, const float *Dskip, const float *h0,
                       void *y, float *h_final, const DtPre &pre, cudaStream_t st);

// --- decode step ---
ssd_status step_launch(const Problem &pr, float *h, const void *x, const void *dt,
                       const float *A, const void *B, const void *C, const float *D,
                       void *y, cudaStream_t st, const DtPre &pre = DtPre());

// Launch accounting: call around every kernel launch (see profile.cu).
void launch_begin(const char *name, cudaStream_t st);
void launch_end(cudaStream_t st);

// Device address of this library's error word on the current device.
unsigned int *device_error_word();

// Clock cycles a pipelined kernel's bounded wait may take before the kernel
// gives up and reports SSD_ERR_TIMEOUT (ssd_set_wait_limit; default ~2 s).
constexpr long long kDefaultWaitCycles = 4000000000LL;
long long wait_limit_cycles();

}  // namespace ssd
