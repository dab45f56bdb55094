// pool.cu -- per-device cache of the runtime's device workspaces, pinned host
// buffers and streams.
//
// A plan allocates a workspace, a pinned read-back buffer and an internal
// stream; applications that solve many problems in a row (every benchmark
// step, every row block) would otherwise pay cudaMalloc / cudaFree (which
// synchronises the device), page pinning and stream creation every time. Freed
// resources go back to this cache (up to kKeepBytes of device memory per
// device) and a later plan of the same or a slightly smaller size reuses them.
// ot_trim_cache() releases everything the cache holds. A resource goes back
// under the device it was made on (the caller names it), whichever device is
// current when it is returned.
#include <atomic>
#include <map>
#include <mutex>
#include <vector>

#include "ot_sinkhorn.h"
#include "ot_sinkhorn_testing.h"
#include "runtime.h"

namespace ot {
namespace {

constexpr int kDevices = 64;
constexpr size_t kKeepBytes = size_t(4) << 30;  // cached device memory per device

struct Pool {
    std::mutex mu;
    std::multimap<size_t, void *> dev[kDevices];
    size_t dev_bytes[kDevices] = {};
    std::multimap<size_t, void *> host;
    std::vector<cudaStream_t> streams[kDevices];
};

Pool &pool() {
    static Pool *p = new Pool();  // never destroyed: resources may be returned at exit
    return *p;
}

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kDevices) return -1;
    return d;
}

// smallest cached block of at least `bytes` and at most twice that
void *take(std::multimap<size_t, void *> &m, size_t bytes, size_t *got) {
    auto it = m.lower_bound(bytes);
    if (it == m.end() || it->first > 2 * bytes + (size_t(1) << 20)) return nullptr;
    void *p = it->second;
    *got = it->first;
    m.erase(it);
    return p;
}

}  // namespace

// Allocation-failure injection for the host-side failure tests (see
// ot_testing_fail_device_allocs): allocations left before one fails, -1 = off.
std::atomic<int> g_fail_countdown{-1};

cudaError_t pool_device_alloc(void **ptr, size_t bytes, size_t *got) {
    int left = g_fail_countdown.load();
    while (left >= 0 && !g_fail_countdown.compare_exchange_weak(left, left - 1)) {
    }
    if (left == 0) {
        *ptr = nullptr;
        return cudaErrorMemoryAllocation;
    }
    const int d = current_device();
    if (d >= 0) {
        Pool &P = pool();
        std::lock_guard<std::mutex> lk(P.mu);
        if (void *p = take(P.dev[d], bytes, got)) {
            P.dev_bytes[d] -= *got;
            *ptr = p;
            return cudaSuccess;
        }
    }
    *got = bytes;
    return cudaMalloc(ptr, bytes);
}

void pool_device_free(void *ptr, size_t bytes, int d) {
    if (!ptr) return;
    if (d >= 0 && d < kDevices) {
        Pool &P = pool();
        std::lock_guard<std::mutex> lk(P.mu);
        if (P.dev_bytes[d] + bytes <= kKeepBytes) {
            P.dev[d].emplace(bytes, ptr);
            P.dev_bytes[d] += bytes;
            return;
        }
    }
    cudaFree(ptr);
}

cudaError_t pool_host_alloc(void **ptr, size_t bytes) {
    {
        Pool &P = pool();
        std::lock_guard<std::mutex> lk(P.mu);
        size_t got = 0;
        if (void *p = take(P.host, bytes, &got)) {
            *ptr = p;
            return cudaSuccess;
        }
    }
    return cudaMallocHost(ptr, bytes);
}

void pool_host_free(void *ptr, size_t bytes) {
    if (!ptr) return;
    Pool &P = pool();
    std::lock_guard<std::mutex> lk(P.mu);
    if (P.host.size() < 64) {
        P.host.emplace(bytes, ptr);
        return;
    }
    cudaFreeHost(ptr);
}

cudaError_t pool_stream(cudaStream_t *s) {
    const int d = current_device();
    if (d >= 0) {
        Pool &P = pool();
        std::lock_guard<std::mutex> lk(P.mu);
        if (!P.streams[d].empty()) {
            *s = P.streams[d].back();
            P.streams[d].pop_back();
            return cudaSuccess;
        }
    }
    return cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
}

void pool_stream_release(cudaStream_t s, int d) {
    if (!s) return;
    if (d >= 0 && d < kDevices) {
        Pool &P = pool();
        std::lock_guard<std::mutex> lk(P.mu);
        if (P.streams[d].size() < 16) {
            P.streams[d].push_back(s);
            return;
        }
    }
    cudaStreamDestroy(s);
}

}  // namespace ot

// Releases every workspace, pinned buffer and stream the library keeps for
// reuse (on all devices it has touched). Plans that are alive are unaffected.
extern "C" void ot_trim_cache(void) {
    using namespace ot;
    Pool &P = pool();
    std::lock_guard<std::mutex> lk(P.mu);
    int prev = 0;
    cudaGetDevice(&prev);
    for (int d = 0; d < kDevices; ++d) {
        if (P.dev[d].empty() && P.streams[d].empty()) continue;
        cudaSetDevice(d);
        for (auto &kv : P.dev[d]) cudaFree(kv.second);
        P.dev[d].clear();
        P.dev_bytes[d] = 0;
        for (cudaStream_t s : P.streams[d]) cudaStreamDestroy(s);
        P.streams[d].clear();
    }
    cudaSetDevice(prev);
    for (auto &kv : P.host) cudaFreeHost(kv.second);
    P.host.clear();
}

// Test hook (include/ot_sinkhorn_testing.h): the device-workspace allocation
// after `after` more successful ones fails as cudaMalloc does when memory runs
// out; a negative value switches the injection off.
extern "C" void ot_testing_fail_device_allocs(int after) {
    ot::g_fail_countdown.store(after < 0 ? -1 : after);
}
