// prof.cu -- optional per-launch timing with CUDA events (off by default).
//
// While enabled on a host thread, every kernel the library launches from that
// thread is bracketed by two cudaEventRecord calls on the launch's own stream,
// so a caller can attribute device time to individual kernels of one ABI call.
#include <vector>

#include "common.cuh"

namespace gdn {
namespace {
struct ProfState {
    bool on = false;
    int cap = 0, n = 0;
    std::vector<cudaEvent_t> ev;
    std::vector<const char*> names;
};
thread_local ProfState g_prof;
}  // namespace

void prof_before(cudaStream_t st) {
    ProfState& p = g_prof;
    if (p.on && p.n < p.cap) cudaEventRecord(p.ev[2 * p.n], st);
}

void prof_after(cudaStream_t st, const char* name) {
    ProfState& p = g_prof;
    if (!p.on) return;
    if (p.n < p.cap) {
        cudaEventRecord(p.ev[2 * p.n + 1], st);
        p.names[p.n] = name;
    }
    ++p.n;
}
}  // namespace gdn

using gdn::g_prof;

extern "C" gdn_status gdn_profile_begin(int capacity) {
    if (capacity < 1 || capacity > (1 << 20)) return GDN_ERR_INVALID_ARG;
    gdn::ProfState& p = g_prof;
    while ((int)p.ev.size() < 2 * capacity) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return GDN_ERR_CUDA;
        p.ev.push_back(e);
    }
    p.names.assign(capacity, nullptr);
    p.cap = capacity;
    p.n = 0;
    p.on = true;
    return GDN_OK;
}

extern "C" int gdn_profile_end(float* ms, const char** names, int capacity) {
    gdn::ProfState& p = g_prof;
    if (!p.on) return -1;
    p.on = false;
    const int n = p.n < p.cap ? p.n : p.cap;
    if (n > 0 && cudaEventSynchronize(p.ev[2 * n - 1]) != cudaSuccess) return -1;
    for (int i = 0; i < n && i < capacity; ++i) {
        float t = 0.f;
        if (cudaEventElapsedTime(&t, p.ev[2 * i], p.ev[2 * i + 1]) != cudaSuccess) t = -1.f;
        if (ms) ms[i] = t;
        if (names) names[i] = p.names[i];
    }
    return p.n;
}
