// Launch accounting and optional per-kernel event timing of the library.
#include <atomic>
#include <mutex>
#include <vector>

#include "saf_common.cuh"

namespace saf {
namespace {

std::atomic<uint64_t> g_launches{0};

struct Record {
    int kid;
    cudaEvent_t start, stop;
};

struct Profile {
    std::mutex mu;
    int max_launches = 0;
    std::vector<Record> recs;
    int open = -1;  // index of the record whose stop event is pending
} g_prof;

const char* kNames[] = {"?", "pattern", "fwd_mma", "dot", "dkdv_mma", "dq_mma",
                        "fwd_tc", "bwd_tc", "(retired)", "dq_convert", "bwd_pre", "group_sum", "pattern_grad", "calibration", "fit"};

void release_locked() {
    for (auto& r : g_prof.recs) {
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    g_prof.recs.clear();
    g_prof.open = -1;
}

}  // namespace

void launch_begin(int kid, cudaStream_t s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if ((int)g_prof.recs.size() >= g_prof.max_launches) return;
    Record r{kid, nullptr, nullptr};
    if (cudaEventCreate(&r.start) != cudaSuccess) return;
    if (cudaEventCreate(&r.stop) != cudaSuccess) {
        cudaEventDestroy(r.start);
        return;
    }
    cudaEventRecord(r.start, s);
    g_prof.recs.push_back(r);
    g_prof.open = (int)g_prof.recs.size() - 1;
}

void launch_end(int kid, cudaStream_t s) {
    (void)kid;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (g_prof.open < 0) return;
    cudaEventRecord(g_prof.recs[g_prof.open].stop, s);
    g_prof.open = -1;
}

}  // namespace saf

extern "C" {

uint64_t saf_launch_count(void) { return saf::g_launches.load(); }

saf_status saf_profile_enable(int max_launches) {
    std::lock_guard<std::mutex> lk(saf::g_prof.mu);
    saf::release_locked();
    saf::g_prof.max_launches = max_launches > 0 ? max_launches : 0;
    saf::g_prof.recs.reserve(saf::g_prof.max_launches);
    return SAF_OK;
}

int saf_profile_read(int* kernel_ids, float* ms, int n) {
    std::lock_guard<std::mutex> lk(saf::g_prof.mu);
    const int avail = (int)saf::g_prof.recs.size();
    for (int i = 0; i < avail && i < n; ++i) {
        auto& r = saf::g_prof.recs[i];
        if (cudaEventSynchronize(r.stop) != cudaSuccess) return -1;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return -1;
        if (kernel_ids) kernel_ids[i] = r.kid;
        if (ms) ms[i] = t;
    }
    return avail;
}

const char* saf_kernel_name(int kernel_id) {
    const int n = (int)(sizeof(saf::kNames) / sizeof(saf::kNames[0]));
    return (kernel_id > 0 && kernel_id < n) ? saf::kNames[kernel_id] : "?";
}

}  // extern "C"
