// ssd_forward_noalloc: the forward pass with its scratch in a fixed array
// compiled into the library, for callers that cannot allocate device memory.
//
// Who needs it: programs that must not allocate on the device once they are
// running. Examples: a serving process that reserves all GPU memory for its
// own pool at start-up, so a cudaMalloc would fail; a real-time loop where an
// allocation's implicit synchronisation or latency is not allowed; a plain C
// caller with no device allocator of its own. ssd_forward's workspace argument
// already lets a caller hand in memory; this entry point is for callers that
// have none to hand in.
//
// The scratch is one file-scope device array of kScratchBytes (32 MiB). Every
// GPU that loads this library holds it until the process exits. Host code may
// not use the array's name as a device address (on the host it is only a
// stand-in symbol), so its device address is looked up with
// cudaGetSymbolAddress, once per device, on that device's first call.
#include <mutex>

#include "internal.h"

namespace ssd {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
void *g_scratch_addr[kMaxDev] = {};
std::mutex g_scratch_mu;

// Device address of g_scratch on the current device (looked up on first use).
ssd_status scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDev)
        return fail(SSD_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the fixed scratch");
        if (!p) return fail(SSD_ERR_CUDA, "cudaGetSymbolAddress returned NULL");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SSD_OK;
}

}  // namespace
}  // namespace ssd

using namespace ssd;

extern "C" ssd_status ssd_forward_noalloc(const void *x, const void *dt, const float *A,
                                          const void *B, const void *C, const float *D,
                                          const float *h0, int chunk, void *y, float *h_final,
                                          const ssd_dims *dims, ssd_stream stream) {
    // Sizes are validated by ssd_forward below; an invalid problem reports 0
    // bytes here and its own error there.
    const size_t need = ssd_forward_workspace_size(dims, chunk);
    if (need > kScratchBytes)
        return fail(SSD_ERR_UNSUPPORTED,
                    "ssd_forward_noalloc: this problem needs %zu bytes of scratch but the "
                    "library's fixed scratch holds %zu; pass a workspace to ssd_forward instead",
                    need, kScratchBytes);
    void *scratch = nullptr;
    const ssd_status s = scratch_address(&scratch);
    if (s != SSD_OK) return s;
    // Every scratch word the forward reads is written earlier in the same
    // call, so nothing needs clearing between calls.
    return ssd_forward(x, dt, A, B, C, D, h0, chunk, y, h_final, dims, scratch, kScratchBytes,
                       stream);
}
