// Launch accounting and optional per-kernel CUDA-event timing.
//
// Every kernel launch of the library goes through launch_begin/launch_end.
// The launch counter is always on. While a profiling window is open
// (ssd_profile_begin .. ssd_profile_end) each launch is bracketed by two CUDA
// events recorded on the launch's own stream, so the measured interval is
// that kernel's execution on that stream.
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace ssd {
namespace {

struct Rec {
    const char *name;
    cudaEvent_t a, b;
};

std::atomic<long long> g_launches{0};
std::mutex g_mu;
bool g_on = false;
bool g_overflow = false;
std::vector<Rec> g_recs;         // records of the open window
std::vector<cudaEvent_t> g_pool; // spare events
size_t g_next = 0;               // records used in the open window
constexpr size_t kMaxRecs = 1 << 16;
thread_local int t_pending = -1;  // record index opened by launch_begin

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

void launch_begin(const char *name, cudaStream_t st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    t_pending = -1;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on) return;
    if (g_next >= kMaxRecs) {
        g_overflow = true;
        return;
    }
    Rec r{name, take_event(), take_event()};
    if (!r.a || !r.b) {
        g_overflow = true;
        return;
    }
    cudaEventRecord(r.a, st);
    if (g_next < g_recs.size()) g_recs[g_next] = r;
    else g_recs.push_back(r);
    t_pending = (int)g_next++;
}

void launch_end(cudaStream_t st) {
    if (t_pending < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_on && (size_t)t_pending < g_next) cudaEventRecord(g_recs[t_pending].b, st);
    t_pending = -1;
}

}  // namespace ssd

using namespace ssd;

extern "C" {

long long ssd_launch_count(void) { return g_launches.load(); }

ssd_status ssd_profile_begin(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (size_t i = 0; i < g_next; ++i) {
        g_pool.push_back(g_recs[i].a);
        g_pool.push_back(g_recs[i].b);
    }
    g_next = 0;
    g_overflow = false;
    g_on = true;
    return SSD_OK;
}

int ssd_profile_end(ssd_kernel_time *out, int max_entries) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_on = false;
    int n = 0;
    for (size_t i = 0; i < g_next; ++i) {
        const Rec &r = g_recs[i];
        if (cudaEventSynchronize(r.b) != cudaSuccess) {
            fail(SSD_ERR_CUDA, "profile event synchronize failed");
            return -1;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            fail(SSD_ERR_CUDA, "profile event elapsed time failed");
            return -1;
        }
        int k = 0;
        while (k < n && strcmp(out[k].name, r.name) != 0) ++k;
        if (k == n) {
            if (n >= max_entries) continue;
            out[n].name = r.name;
            out[n].launches = 0;
            out[n].total_ms = 0.0;
            ++n;
        }
        out[k].launches += 1;
        out[k].total_ms += ms;
    }
    if (g_overflow) {
        fail(SSD_ERR_NO_MEMORY, "profile window overflowed; some launches were not timed");
        return -1;
    }
    return n;
}

}  // extern "C"
