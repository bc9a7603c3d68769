// libssd C ABI: argument validation, workspace handling and dispatch.
// The entry points are declared, with their contracts, in include/ssd.h.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace ssd {
namespace {

thread_local char g_msg[512] = "";

// Device-side error word (bounded waits that give up set it); one copy per
// device that loads the library.
__device__ unsigned int g_err_word = 0;

constexpr int kMaxDevices = 64;
unsigned int *g_err_addr[kMaxDevices] = {};
std::mutex g_err_mu;

std::atomic<long long> g_wait_limit{0};  // 0: kDefaultWaitCycles

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ssd_status check_dims(const ssd_dims *d, bool need_seq) {
    if (!d) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    if (d->reserved != 0) return fail(SSD_ERR_INVALID_ARG, "dims.reserved must be 0");
    if (d->dtype != SSD_F32 && d->dtype != SSD_BF16)
        return fail(SSD_ERR_INVALID_ARG, "dims.dtype %d is not SSD_F32 or SSD_BF16", d->dtype);
    if (d->batch < 1 || d->nheads < 1 || d->ngroups < 1 || d->headdim < 1 || d->dstate < 1)
        return fail(SSD_ERR_INVALID_ARG,
                    "sizes must be positive (batch %lld, nheads %lld, ngroups %lld, headdim "
                    "%lld, dstate %lld)",
                    (long long)d->batch, (long long)d->nheads, (long long)d->ngroups,
                    (long long)d->headdim, (long long)d->dstate);
    if (need_seq && d->seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "seqlen %lld < 0", (long long)d->seqlen);
    if (d->nheads % d->ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "nheads %lld is not a multiple of ngroups %lld",
                    (long long)d->nheads, (long long)d->ngroups);
    if (d->headdim % 16 != 0 || d->headdim > 128)
        return fail(SSD_ERR_UNSUPPORTED, "headdim %lld: supported 16..128 in steps of 16",
                    (long long)d->headdim);
    if (d->dstate % 16 != 0 || d->dstate > 256)
        return fail(SSD_ERR_UNSUPPORTED, "dstate %lld: supported 16..256 in steps of 16",
                    (long long)d->dstate);
    if (d->batch > 65535 || d->nheads > 65535)
        return fail(SSD_ERR_UNSUPPORTED, "batch and nheads are limited to 65535");
    // 32-bit grid limits and 64-bit indexing headroom
    if ((double)d->batch * d->nheads > 2.0e9)
        return fail(SSD_ERR_UNSUPPORTED, "batch * nheads too large");
    if (need_seq && d->seqlen > (int64_t)1 << 30)
        return fail(SSD_ERR_UNSUPPORTED, "seqlen above 2^30");
    return SSD_OK;
}

bool chunk_ok(int chunk) {
    return chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128 || chunk == 256;
}

Problem make_problem(const ssd_dims *d, int chunk) {
    Problem p;
    p.batch = d->batch;
    p.seqlen = d->seqlen;
    p.nheads = d->nheads;
    p.headdim = d->headdim;
    p.dstate = d->dstate;
    p.ngroups = d->ngroups;
    p.dtype = d->dtype;
    p.chunk = chunk;
    return p;
}

// Forward path selection. LIBSSD_FORWARD_PATH=simt forces the CUDA-core path
// and =tc requires the tensor-core path (for testing one against the other);
// unset, the tensor-core path serves every problem it supports.
enum Path { kAuto = 0, kSimt = 1, kTc = 2 };
int path_override() {
    static int v = -1;
    if (v < 0) {
        const char *e = getenv("LIBSSD_FORWARD_PATH");
        v = (e && !strcmp(e, "simt")) ? kSimt : (e && !strcmp(e, "tc")) ? kTc : kAuto;
    }
    return v;
}

bool use_tc(const Problem &pr) { return path_override() != kSimt && tc_supported(pr); }

size_t workspace_bytes(const Problem &pr) {
    return use_tc(pr) ? tc_workspace_bytes(pr) : simt_workspace_bytes(pr);
}

// ssd_options -> the kernels' DtPre (NULL: none), after validation.
ssd_status read_options(const ssd_options *o, DtPre *pre) {
    *pre = DtPre();
    if (!o) return SSD_OK;
    for (int i = 0; i < 4; ++i)
        if (o->reserved[i] != 0)
            return fail(SSD_ERR_INVALID_ARG, "options.reserved[%d] must be 0", i);
    if (o->discretization != SSD_DISC_EULER && o->discretization != SSD_DISC_ZOH)
        return fail(SSD_ERR_INVALID_ARG, "options.discretization %d is not SSD_DISC_EULER or "
                                         "SSD_DISC_ZOH", o->discretization);
    if (o->dt_bias && !aligned(o->dt_bias, 4))
        return fail(SSD_ERR_INVALID_ARG, "options.dt_bias is misaligned");
    if (!(o->dt_max <= 0.f) && !(o->dt_max > 0.f))
        return fail(SSD_ERR_INVALID_ARG, "options.dt_max is NaN");
    if (o->dt_max > 0.f && !(o->dt_min >= 0.f && o->dt_min <= o->dt_max))
        return fail(SSD_ERR_INVALID_ARG, "options: need 0 <= dt_min <= dt_max (got %g, %g)",
                    (double)o->dt_min, (double)o->dt_max);
    pre->bias = o->dt_bias;
    pre->softplus = o->dt_softplus != 0;
    pre->zoh = o->discretization == SSD_DISC_ZOH;
    pre->dt_min = o->dt_max > 0.f ? o->dt_min : 0.f;
    pre->dt_max = o->dt_max > 0.f ? o->dt_max : 0.f;
    return SSD_OK;
}

}  // namespace

ssd_status fail(ssd_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return s;
}

ssd_status cuda_fail(cudaError_t e, const char *what) {
    return fail(SSD_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

unsigned int *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return nullptr;
        g_err_addr[dev] = static_cast<unsigned int *>(p);
    }
    return g_err_addr[dev];
}

long long wait_limit_cycles() {
    const long long v = g_wait_limit.load(std::memory_order_relaxed);
    return v > 0 ? v : kDefaultWaitCycles;
}

}  // namespace ssd

using namespace ssd;

extern "C" {

void ssd_set_wait_limit(long long cycles) {
    g_wait_limit.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed);
}

int ssd_abi_version(void) { return SSD_ABI_VERSION; }

const char *ssd_last_error(void) { return g_msg; }

size_t ssd_forward_workspace_size(const ssd_dims *dims, int chunk) {
    if (check_dims(dims, true) != SSD_OK) return 0;
    if (!chunk_ok(chunk)) {
        fail(SSD_ERR_UNSUPPORTED, "chunk %d: supported 16, 32, 64, 128, 256", chunk);
        return 0;
    }
    return workspace_bytes(make_problem(dims, chunk));
}

ssd_status ssd_forward(const void *x, const void *dt, const float *A, const void *B,
                       const void *C, const float *D, const float *h0, int chunk, void *y,
                       float *h_final, const ssd_dims *dims, void *workspace,
                       size_t workspace_bytes_given, ssd_stream stream) {
    return ssd_forward_ex(x, dt, A, B, C, D, h0, chunk, y, h_final, dims, nullptr, workspace,
                          workspace_bytes_given, stream);
}

ssd_status ssd_forward_ex(const void *x, const void *dt, const float *A, const void *B,
                          const void *C, const float *D, const float *h0, int chunk, void *y,
                          float *h_final, const ssd_dims *dims, const ssd_options *opts,
                          void *workspace, size_t workspace_bytes_given, ssd_stream stream) {
    ssd_status s = check_dims(dims, true);
    if (s != SSD_OK) return s;
    DtPre pre;
    if ((s = read_options(opts, &pre)) != SSD_OK) return s;
    if (!chunk_ok(chunk))
        return fail(SSD_ERR_UNSUPPORTED, "chunk %d: supported 16, 32, 64, 128, 256", chunk);
    const Problem pr = make_problem(dims, chunk);
    const size_t esz = pr.dtype == SSD_F32 ? 4 : 2;
    if (!A) return fail(SSD_ERR_INVALID_ARG, "A is NULL");
    if (pr.seqlen > 0 && (!x || !dt || !B || !C || !y))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, B, C and y must be non-NULL");
    const void *p16[] = {x, B, C, y, h0, h_final};
    const char *n16[] = {"x", "B", "C", "y", "h0", "h_final"};
    for (int i = 0; i < 6; ++i)
        if (p16[i] && !aligned(p16[i], 16))
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", n16[i]);
    if (dt && !aligned(dt, esz)) return fail(SSD_ERR_INVALID_ARG, "dt is misaligned");
    if (!aligned(A, 4) || (D && !aligned(D, 4)))
        return fail(SSD_ERR_INVALID_ARG, "A or D is misaligned");
    if (y && (y == x || y == dt || y == B || y == C))
        return fail(SSD_ERR_INVALID_ARG, "y aliases an input");
    const size_t need = workspace_bytes(pr);
    if (workspace) {
        if (workspace_bytes_given < need)
            return fail(SSD_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed",
                        workspace_bytes_given, need);
        if (!aligned(workspace, 256))
            return fail(SSD_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void *ws = workspace;
    bool owned = false;
    if (!ws && need > 0) {
        const cudaError_t e = cudaMallocAsync(&ws, need, st);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(SSD_ERR_NO_MEMORY, "cudaMallocAsync of %zu workspace bytes: %s", need,
                        cudaGetErrorString(e));
        }
        owned = true;
    }
    if (path_override() == kTc && !tc_supported(pr) && pr.seqlen > 0) {
        s = fail(SSD_ERR_UNSUPPORTED, "LIBSSD_FORWARD_PATH=tc but the tensor-core path needs "
                                      "bf16, headdim 64, dstate 64/128/256 and chunk 128/256");
    } else if (use_tc(pr)) {
        s = tc_forward(pr, x, dt, A, B, C, D, h0, y, h_final, ws, st, pre);
    } else {
        s = simt_forward(pr, x, dt, A, B, C, D, h0, y, h_final, ws, st, pre);
    }
    if (owned) {
        const cudaError_t e = cudaFreeAsync(ws, st);
        if (e != cudaSuccess && s == SSD_OK) s = cuda_fail(e, "cudaFreeAsync of the workspace");
    }
    return s;
}

ssd_status ssd_step(float *h, const void *x, const void *dt, const float *A, const void *B,
                    const void *C, const float *D, void *y, const ssd_dims *dims,
                    ssd_stream stream) {
    return ssd_step_ex(h, x, dt, A, B, C, D, y, dims, nullptr, stream);
}

ssd_status ssd_step_ex(float *h, const void *x, const void *dt, const float *A, const void *B,
                       const void *C, const float *D, void *y, const ssd_dims *dims,
                       const ssd_options *opts, ssd_stream stream) {
    ssd_status s = check_dims(dims, false);
    if (s != SSD_OK) return s;
    DtPre pre;
    if ((s = read_options(opts, &pre)) != SSD_OK) return s;
    const Problem pr = make_problem(dims, 0);
    const size_t esz = pr.dtype == SSD_F32 ? 4 : 2;
    if (!h || !x || !dt || !A || !B || !C || !y)
        return fail(SSD_ERR_INVALID_ARG, "h, x, dt, A, B, C and y must be non-NULL");
    const void *p16[] = {h, B, C};
    const char *n16[] = {"h", "B", "C"};
    for (int i = 0; i < 3; ++i)
        if (!aligned(p16[i], 16))
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", n16[i]);
    if (!aligned(x, esz) || !aligned(dt, esz) || !aligned(y, esz) || !aligned(A, 4) ||
        (D && !aligned(D, 4)))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, y, A or D is misaligned");
    if (y == (void *)h || y == x || y == dt || y == B || y == C)
        return fail(SSD_ERR_INVALID_ARG, "y aliases h or an input");
    return step_launch(pr, h, x, dt, A, B, C, D, y, reinterpret_cast<cudaStream_t>(stream), pre);
}

size_t ssd_forward_state_workspace_size(const ssd_dims *dims, int chunk) {
    if (check_dims(dims, true) != SSD_OK) return 0;
    if (!chunk_ok(chunk)) {
        fail(SSD_ERR_UNSUPPORTED, "chunk %d: supported 16, 32, 64, 128, 256", chunk);
        return 0;
    }
    const Problem pr = make_problem(dims, chunk);
    return (use_tc(pr) && pr.seqlen > 0) ? tc_state_workspace_bytes(pr)
                                         : simt_workspace_bytes(pr);
}

ssd_status ssd_forward_state(const void *x, const void *dt, const float *A, const void *B,
                             int chunk, float *state_out, float *decay_out, const ssd_dims *dims,
                             const ssd_options *opts, void *workspace,
                             size_t workspace_bytes_given, ssd_stream stream) {
    ssd_status s = check_dims(dims, true);
    if (s != SSD_OK) return s;
    if (!chunk_ok(chunk))
        return fail(SSD_ERR_UNSUPPORTED, "chunk %d: supported 16, 32, 64, 128, 256", chunk);
    DtPre pre;
    if ((s = read_options(opts, &pre)) != SSD_OK) return s;
    const Problem pr = make_problem(dims, chunk);
    const size_t esz = pr.dtype == SSD_F32 ? 4 : 2;
    if (!A || !state_out || !decay_out)
        return fail(SSD_ERR_INVALID_ARG, "A, state_out and decay_out must be non-NULL");
    if (pr.seqlen > 0 && (!x || !dt || !B))
        return fail(SSD_ERR_INVALID_ARG, "x, dt and B must be non-NULL");
    const void *p16[] = {x, B, state_out};
    const char *n16[] = {"x", "B", "state_out"};
    for (int i = 0; i < 3; ++i)
        if (p16[i] && !aligned(p16[i], 16))
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", n16[i]);
    if ((dt && !aligned(dt, esz)) || !aligned(A, 4) || !aligned(decay_out, 4))
        return fail(SSD_ERR_INVALID_ARG, "dt, A or decay_out is misaligned");
    const bool tc = use_tc(pr) && pr.seqlen > 0;
    const size_t need = tc ? tc_state_workspace_bytes(pr) : simt_workspace_bytes(pr);
    if (workspace) {
        if (workspace_bytes_given < need)
            return fail(SSD_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed",
                        workspace_bytes_given, need);
        if (!aligned(workspace, 256))
            return fail(SSD_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void *ws = workspace;
    bool owned = false;
    if (!ws && need > 0) {
        const cudaError_t e = cudaMallocAsync(&ws, need, st);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(SSD_ERR_NO_MEMORY, "cudaMallocAsync of %zu workspace bytes: %s", need,
                        cudaGetErrorString(e));
        }
        owned = true;
    }
    s = tc ? tc_state(pr, x, dt, A, B, state_out, decay_out, ws, st, pre)
           : simt_state(pr, x, dt, A, B, state_out, decay_out, ws, st, pre);
    if (owned) {
        const cudaError_t e = cudaFreeAsync(ws, st);
        if (e != cudaSuccess && s == SSD_OK) s = cuda_fail(e, "cudaFreeAsync of the workspace");
    }
    return s;
}

ssd_status ssd_state_chain(const float *states, const float *decays, int nparts, int part,
                           const float *h0, float *h_in, float *h_total, const ssd_dims *dims,
                           ssd_stream stream) {
    ssd_status s = check_dims(dims, false);
    if (s != SSD_OK) return s;
    if (nparts < 1 || part < 0 || part >= nparts)
        return fail(SSD_ERR_INVALID_ARG, "part %d of %d pieces", part, nparts);
    if (!states || !decays || (!h_in && !h_total))
        return fail(SSD_ERR_INVALID_ARG, "states, decays and one of h_in, h_total are required");
    const void *p16[] = {states, h0, h_in, h_total};
    const char *n16[] = {"states", "h0", "h_in", "h_total"};
    for (int i = 0; i < 4; ++i)
        if (p16[i] && !aligned(p16[i], 16))
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", n16[i]);
    if (!aligned(decays, 4)) return fail(SSD_ERR_INVALID_ARG, "decays is misaligned");
    return state_chain_launch(states, decays, h0, h_in, h_total, dims->batch, dims->nheads,
                              (int)(dims->headdim * dims->dstate / 4), nparts, part,
                              reinterpret_cast<cudaStream_t>(stream));
}

ssd_status ssd_selective_scan(const void *x, const void *dt, const float *A, const void *B,
                              const void *C, const float *Dskip, const float *h0, void *y,
                              float *h_final, const ssd_dims *dims, const ssd_options *opts,
                              ssd_stream stream) {
    if (!dims) return fail(SSD_ERR_INVALID_ARG, "dims is NULL");
    if (dims->reserved != 0) return fail(SSD_ERR_INVALID_ARG, "dims.reserved must be 0");
    if (dims->dtype != SSD_F32 && dims->dtype != SSD_BF16)
        return fail(SSD_ERR_INVALID_ARG, "dims.dtype %d is not SSD_F32 or SSD_BF16", dims->dtype);
    if (dims->batch < 1 || dims->nheads < 1 || dims->ngroups < 1 || dims->seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "sizes must be positive (seqlen >= 0)");
    if (dims->headdim != 1)
        return fail(SSD_ERR_INVALID_ARG, "selective scan: headdim must be 1 (one channel per "
                                         "head), got %lld", (long long)dims->headdim);
    if (dims->nheads % dims->ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "channels %lld not a multiple of ngroups %lld",
                    (long long)dims->nheads, (long long)dims->ngroups);
    if (!scan_supported_dstate(dims->dstate))
        return fail(SSD_ERR_UNSUPPORTED, "selective scan: dstate %lld: supported 4, 8, 16",
                    (long long)dims->dstate);
    if (dims->batch > 65535 || (double)dims->batch * dims->seqlen * dims->nheads > 4.0e18)
        return fail(SSD_ERR_UNSUPPORTED, "batch above 65535");
    DtPre pre;
    ssd_status s = read_options(opts, &pre);
    if (s != SSD_OK) return s;
    const Problem pr = make_problem(dims, 0);
    const size_t esz = pr.dtype == SSD_F32 ? 4 : 2;
    if (!A) return fail(SSD_ERR_INVALID_ARG, "A is NULL");
    if (pr.seqlen > 0 && (!x || !dt || !B || !C || !y))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, B, C and y must be non-NULL");
    // B and C rows are read 4 elements at a time
    if ((B && !aligned(B, 4 * esz)) || (C && !aligned(C, 4 * esz)))
        return fail(SSD_ERR_INVALID_ARG, "B and C must be %zu-byte aligned", 4 * esz);
    if ((x && !aligned(x, esz)) || (dt && !aligned(dt, esz)) || (y && !aligned(y, esz)) ||
        !aligned(A, 4) || (Dskip && !aligned(Dskip, 4)) || (h0 && !aligned(h0, 4)) ||
        (h_final && !aligned(h_final, 4)))
        return fail(SSD_ERR_INVALID_ARG, "a pointer is misaligned for its type");
    if (y && (y == x || y == dt || y == B || y == C))
        return fail(SSD_ERR_INVALID_ARG, "y aliases an input");
    return scan_launch(pr, x, dt, A, B, C, Dskip, h0, y, h_final, pre,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t ssd_backward_workspace_size(const ssd_dims *dims) {
    if (check_dims(dims, true) != SSD_OK) return 0;
    const Problem pr = make_problem(dims, 64);
    if (backward_chunk(pr) == 0) {
        fail(SSD_ERR_UNSUPPORTED, "backward: headdim x dstate too large");
        return 0;
    }
    return backward_workspace_bytes(pr);
}

ssd_status ssd_backward(const void *x, const void *dt, const float *A, const void *B,
                        const void *C, const float *D, const float *h0, const void *dy,
                        const float *dh_final, float *dx, float *ddt, float *dA, float *dB,
                        float *dC, float *dD, float *dh0, const ssd_dims *dims, void *workspace,
                        size_t workspace_bytes_given, ssd_stream stream) {
    ssd_status s = check_dims(dims, true);
    if (s != SSD_OK) return s;
    const Problem pr = make_problem(dims, 64);
    if (backward_chunk(pr) == 0)
        return fail(SSD_ERR_UNSUPPORTED, "backward: headdim %lld x dstate %lld too large",
                    (long long)pr.headdim, (long long)pr.dstate);
    if (!A || !dA || !dD) return fail(SSD_ERR_INVALID_ARG, "A, dA and dD are required");
    if (pr.seqlen > 0 && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, B, C, dy and the gradients dx, ddt, dB, dC "
                                         "must be non-NULL");
    const size_t esz = pr.dtype == SSD_F32 ? 4 : 2;
    // the tensor-core kernels load x, dy, B and C as tiles and write dx, dB
    // and dC sixteen bytes at a time
    const void *p16[] = {x, B, C, dy, dx, dB, dC, h0, dh_final, dh0};
    const char *n16[] = {"x", "B", "C", "dy", "dx", "dB", "dC", "h0", "dh_final", "dh0"};
    for (int i = 0; i < 10; ++i)
        if (p16[i] && !aligned(p16[i], 16))
            return fail(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", n16[i]);
    if ((dt && !aligned(dt, esz)) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (ddt && !aligned(ddt, 4)) || !aligned(dA, 4) || !aligned(dD, 4))
        return fail(SSD_ERR_INVALID_ARG, "a pointer is misaligned for its type");
    const size_t need = backward_workspace_bytes(pr);
    if (workspace) {
        if (workspace_bytes_given < need)
            return fail(SSD_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed",
                        workspace_bytes_given, need);
        if (!aligned(workspace, 256))
            return fail(SSD_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void *ws = workspace;
    bool owned = false;
    if (!ws && need > 0) {
        const cudaError_t e = cudaMallocAsync(&ws, need, st);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(SSD_ERR_NO_MEMORY, "cudaMallocAsync of %zu workspace bytes: %s", need,
                        cudaGetErrorString(e));
        }
        owned = true;
    }
    s = backward_launch(pr, x, dt, A, B, C, D, h0, dy, dh_final, dx, ddt, dA, dB, dC, dD, dh0,
                        ws, st);
    if (owned) {
        const cudaError_t e = cudaFreeAsync(ws, st);
        if (e != cudaSuccess && s == SSD_OK) s = cuda_fail(e, "cudaFreeAsync of the workspace");
    }
    return s;
}

ssd_status ssd_device_status(ssd_stream stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int *w = device_error_word();
    if (!w) return fail(SSD_ERR_CUDA, "cannot locate the device error word");
    unsigned int v = 0;
    e = cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpy(w, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
        return fail(SSD_ERR_TIMEOUT, "a kernel's bounded wait gave up (code 0x%x)", v);
    }
    return SSD_OK;
}

}  // extern "C"
