// ua_profile.cu -- optional per-kernel timing: when enabled, every libua kernel launch is
// bracketed by a pair of CUDA events recorded on the launch's stream.  Reading the table
// synchronises on the recorded events and aggregates launches and total time per kernel.
#include <string.h>

#include <mutex>

#include "ua_common.cuh"
#include "ua_profile.h"

namespace ua {
namespace {

constexpr int kMaxRecords = 8192;

struct Record {
    const char* name;
    cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_enabled = false;
Record g_rec[kMaxRecords];
int g_n = 0;
int g_created = 0;
bool g_overflow = false;

}  // namespace

ProfileScope::ProfileScope(const char* name, cudaStream_t s) : idx_(-1), stream_(s) {
    if (!g_enabled) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_n >= kMaxRecords) { g_overflow = true; return; }
    Record& r = g_rec[g_n];
    if (g_n >= g_created) {
        if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return;
        ++g_created;
    }
    r.name = name;
    idx_ = g_n++;
    cudaEventRecord(r.start, stream_);
}

ProfileScope::~ProfileScope() {
    if (idx_ >= 0) cudaEventRecord(g_rec[idx_].stop, stream_);
}

}  // namespace ua

using namespace ua;

extern "C" {

ua_status ua_profile_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_enabled = enable != 0;
    return UA_OK;
}

ua_status ua_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_n = 0;
    g_overflow = false;
    return UA_OK;
}

ua_status ua_profile_read(ua_kernel_time* out, int max_entries, int* n_entries) {
    if (!n_entries || (max_entries > 0 && !out)) return UA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    int m = 0;
    for (int i = 0; i < g_n; ++i) {
        if (cudaEventSynchronize(g_rec[i].stop) != cudaSuccess) return UA_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_rec[i].start, g_rec[i].stop) != cudaSuccess) return UA_ERR_CUDA;
        int k = 0;
        while (k < m && strcmp(out[k].name, g_rec[i].name) != 0) ++k;
        if (k == m) {
            if (m >= max_entries) continue;
            out[m].name = g_rec[i].name;
            out[m].launches = 0;
            out[m].total_ms = 0.0;
            ++m;
        }
        out[k].launches += 1;
        out[k].total_ms += ms;
    }
    *n_entries = m;
    return g_overflow ? UA_ERR_CAPACITY : UA_OK;
}

}  // extern "C"
