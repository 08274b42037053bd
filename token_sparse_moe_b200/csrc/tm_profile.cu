// tm_profile.cu -- launch counting and optional per-kernel CUDA-event timing.
//
// Every kernel launch of the library goes through a ProfileScope.  The launch
// counter is always kept; when profiling is on, an event pair is recorded on the
// launching stream around the launch and folded into per-kernel totals by
// tm_profile_stop.  Events come from a pool that grows on demand and is reused.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "tm.h"
#include "tm_internal.h"

namespace tml {

namespace {
struct Rec {
    const char* name;
    int ev;  // index of the start event; end event is ev + 1
};
std::mutex g_mu;
bool g_on = false;
unsigned long long g_launches = 0;
std::vector<cudaEvent_t> g_pool;
std::vector<Rec> g_recs;
size_t g_next = 0;
char g_last_err[256] = "";
int g_debug_sync = -1;   // TM_DEBUG_SYNC=1: synchronise after every launch and name a failing kernel

int take_pair() {
    if (g_next + 2 > g_pool.size()) {
        for (int i = 0; i < 256; ++i) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return -1;
            g_pool.push_back(e);
        }
    }
    const int i = (int)g_next;
    g_next += 2;
    return i;
}
}  // namespace

void note_cuda_error(const char* where, cudaError_t e) {
    if (e == cudaSuccess) return;
    std::lock_guard<std::mutex> lk(g_mu);
    snprintf(g_last_err, sizeof(g_last_err), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

ProfileScope::ProfileScope(const char* name, cudaStream_t st) : st_(st), ev_(-1), name_(name) {
    std::lock_guard<std::mutex> lk(g_mu);
    ++g_launches;
    if (!g_on) return;
    ev_ = take_pair();
    if (ev_ < 0) return;
    cudaEventRecord(g_pool[ev_], st);
    g_recs.push_back(Rec{name, ev_});
}

ProfileScope::~ProfileScope() {
    if (ev_ >= 0) {
        std::lock_guard<std::mutex> lk(g_mu);
        cudaEventRecord(g_pool[ev_ + 1], st_);
    }
    if (g_debug_sync < 0) {
        const char* v = getenv("TM_DEBUG_SYNC");
        g_debug_sync = (v && v[0] == '1') ? 1 : 0;
    }
    if (g_debug_sync == 1) {
        cudaError_t e = cudaStreamSynchronize(st_);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) {
            note_cuda_error(name_, e);
            fprintf(stderr, "tm: kernel %s failed: %s\n", name_, cudaGetErrorString(e));
        }
    }
}

}  // namespace tml

using namespace tml;

extern "C" {

const char* tm_last_cuda_error(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_last_err;
}

unsigned long long tm_launch_count(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_launches;
}

tm_status tm_profile_start(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_recs.clear();
    g_next = 0;
    g_on = true;
    return TM_OK;
}

tm_status tm_profile_stop(tm_kernel_time* out, int max_entries, int* n_entries) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_on = false;
    if (n_entries) *n_entries = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return TM_ERR_CUDA;
    int n = 0;
    for (const Rec& r : g_recs) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_pool[r.ev], g_pool[r.ev + 1]) != cudaSuccess) return TM_ERR_CUDA;
        int j = 0;
        while (j < n && strncmp(out[j].name, r.name, sizeof(out[j].name)) != 0) ++j;
        if (j == n) {
            if (!out || n >= max_entries) continue;
            memset(&out[j], 0, sizeof(out[j]));
            strncpy(out[j].name, r.name, sizeof(out[j].name) - 1);
            ++n;
        }
        out[j].launches += 1;
        out[j].total_ms += ms;
    }
    if (n_entries) *n_entries = n;
    g_recs.clear();
    g_next = 0;
    return TM_OK;
}

}  // extern "C"
