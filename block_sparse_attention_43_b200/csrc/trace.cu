// trace.cu -- optional per-kernel CUDA-event timing behind msa_trace_enable /
// msa_trace_read (include/msa.h).  Host code only.
#include <mutex>
#include <vector>

#include "msa.h"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kPool = 4096;

struct Rec {
    const char *name;
    int slot;
};

std::mutex g_mu;
bool g_on = false;
std::vector<cudaEvent_t> g_ev;     // 2 * kPool events: begin, end per slot
std::vector<Rec> g_recs;
int g_open = -1;                   // slot of the launch being recorded

}  // namespace

TraceScope::TraceScope(cudaStream_t s, const char *name) : stream_(s), slot_(-1) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_on || static_cast<int>(g_recs.size()) >= kPool) return;
    slot_ = static_cast<int>(g_recs.size());
    if (cudaEventRecord(g_ev[2 * slot_], s) != cudaSuccess) { slot_ = -1; return; }
    g_recs.push_back({name, slot_});
    g_open = slot_;
}

TraceScope::~TraceScope() {
    if (slot_ < 0) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_on && slot_ < static_cast<int>(g_recs.size())) cudaEventRecord(g_ev[2 * slot_ + 1], stream_);
    g_open = -1;
}

}  // namespace msa

using namespace msa;

extern "C" {

msa_status_t msa_trace_enable(int on) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (on && g_ev.empty()) {
        g_ev.resize(2 * kPool);
        for (auto &e : g_ev)
            if (cudaEventCreate(&e) != cudaSuccess) {
                g_ev.clear();
                return MSA_ERR_CUDA;
            }
    }
    g_on = on != 0;
    g_recs.clear();
    return MSA_OK;
}

int msa_trace_read(const char **names, float *ms, int max_entries) {
    std::lock_guard<std::mutex> lock(g_mu);
    int n = 0;
    int rc = 0;
    for (const Rec &r : g_recs) {
        if (n >= max_entries) break;
        if (cudaEventSynchronize(g_ev[2 * r.slot + 1]) != cudaSuccess) { rc = -1; break; }
        float t = 0.f;
        if (cudaEventElapsedTime(&t, g_ev[2 * r.slot], g_ev[2 * r.slot + 1]) != cudaSuccess) {
            rc = -1;
            break;
        }
        if (names) names[n] = r.name;
        if (ms) ms[n] = t;
        ++n;
    }
    g_recs.clear();
    return rc < 0 ? -1 : n;
}

}  // extern "C"
