// Per-kernel launch counts and (optionally) CUDA-event device times.
// Events are recorded on the launching stream, so the times are those of the
// kernels themselves in stream order; reading them synchronises the events.
#include <cstring>
#include <mutex>
#include <vector>

#include "sata_internal.h"

namespace sata {

int64_t g_opt_time_kernels = 0;

namespace {

struct Pending {
    int id;
    cudaEvent_t start, stop;
};

std::mutex g_mu;
int64_t g_launches[kNumKernels] = {};
double g_ms[kNumKernels] = {};
std::vector<Pending> g_pending;
thread_local cudaEvent_t t_start[kNumKernels] = {};

const char *const kNames[kNumKernels] = {
    "decode_stream", "decode_finish", "simt_scan", "simt_finish",
    "tc_prep", "tc_scan", "tc_finish", "tc_reduce",
    "bwd_r", "bwd_q_scan", "bwd_kv_scan", "bwd_finish", "state_add", "bwd_tc_prep", "bwd_tc_scan",
    "bwd_tc_finish", "tc_stats", "tc_state_stats", "bwd_tc_r",
};

void drain_locked() {
    for (auto &p : g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.stop) == cudaSuccess &&
            cudaEventElapsedTime(&ms, p.start, p.stop) == cudaSuccess)
            g_ms[p.id] += ms;
        cudaEventDestroy(p.start);
        cudaEventDestroy(p.stop);
    }
    g_pending.clear();
}

}  // namespace

const char *kernel_name(int id) { return (id >= 0 && id < kNumKernels) ? kNames[id] : "?"; }

void launch_begin(int id, cudaStream_t s) {
    t_start[id] = nullptr;
    if (!g_opt_time_kernels) return;
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    if (cudaEventRecord(e, s) != cudaSuccess) {
        cudaEventDestroy(e);
        return;
    }
    t_start[id] = e;
}

void launch_end(int id, cudaStream_t s) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_launches[id] += 1;
    cudaEvent_t st = t_start[id];
    t_start[id] = nullptr;
    if (!st) return;
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess || cudaEventRecord(e, s) != cudaSuccess) {
        cudaEventDestroy(st);
        return;
    }
    g_pending.push_back({id, st, e});
    if (g_pending.size() > 4096) drain_locked();
}

}  // namespace sata

using namespace sata;

extern "C" {

int sata_kernel_stats(sata_kernel_stat *out, int max_entries, int *n_out) {
    if (!n_out || max_entries < 0 || (max_entries > 0 && !out)) return SATA_EINVAL;
    std::lock_guard<std::mutex> lk(g_mu);
    drain_locked();
    int n = 0;
    for (int id = 0; id < kNumKernels; ++id) {
        if (!g_launches[id]) continue;
        if (n < max_entries) {
            std::memset(out[n].name, 0, sizeof(out[n].name));
            std::strncpy(out[n].name, kNames[id], sizeof(out[n].name) - 1);
            out[n].launches = g_launches[id];
            out[n].ms = g_ms[id];
        }
        ++n;
    }
    *n_out = n < max_entries ? n : max_entries;
    return SATA_OK;
}

int sata_reset_kernel_stats(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    drain_locked();
    for (int id = 0; id < kNumKernels; ++id) {
        g_launches[id] = 0;
        g_ms[id] = 0.0;
    }
    return SATA_OK;
}

}  // extern "C"
