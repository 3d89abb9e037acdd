// trace.cu -- optional per-kernel device timing.  When enabled, every kernel
// launch of the library is bracketed by two CUDA events recorded on the
// launch stream; a report aggregates the elapsed device time and the launch
// count per kernel name (prefixed by the phase of the entry point that
// launched it, e.g. "dense/score_tc").  Disabled by default: then a launch
// costs one branch.
#include <mutex>
#include <stdio.h>
#include <string.h>
#include <string>
#include <vector>

#include "../../include/idx.h"
#include "internal.h"

namespace idx {

namespace {

struct Rec {
    std::string name;
    cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
thread_local const char *g_phase = "";

cudaEvent_t get_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

TracePhase::TracePhase(const char *p) : prev(g_phase) { g_phase = p; }
TracePhase::~TracePhase() { g_phase = prev; }

TraceScope::TraceScope(const char *name, cudaStream_t st) : st_(st), idx_(-1) {
    if (!g_on) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Rec r;
    r.name = std::string(g_phase) + (g_phase[0] ? "/" : "") + name;
    r.a = get_event();
    r.b = get_event();
    cudaEventRecord(r.a, st_);
    g_recs.push_back(r);
    idx_ = (int)g_recs.size() - 1;
}

TraceScope::~TraceScope() {
    if (idx_ < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (idx_ < (int)g_recs.size()) cudaEventRecord(g_recs[idx_].b, st_);
}

}  // namespace idx

using namespace idx;

extern "C" {

int idx_trace_enable(int on) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (on) {  // a new record; stopping keeps the current one for the report
        for (auto &r : g_recs) {
            g_pool.push_back(r.a);
            g_pool.push_back(r.b);
        }
        g_recs.clear();
    }
    g_on = on != 0;
    return 0;
}

long long idx_trace_report(char *buf, size_t len) {
    std::lock_guard<std::mutex> lk(g_mu);
    struct Agg {
        std::string name;
        long long n;
        double ms;
    };
    std::vector<Agg> agg;
    for (auto &r : g_recs) {
        if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
        bool found = false;
        for (auto &x : agg)
            if (x.name == r.name) {
                x.n += 1;
                x.ms += ms;
                found = true;
                break;
            }
        if (!found) agg.push_back({r.name, 1, (double)ms});
    }
    std::string out;
    char line[512];
    for (auto &x : agg) {
        snprintf(line, sizeof line, "%s %lld %.6f\n", x.name.c_str(), x.n, x.ms);
        out += line;
    }
    if (buf && len) {
        size_t n = out.size() < len - 1 ? out.size() : len - 1;
        memcpy(buf, out.data(), n);
        buf[n] = 0;
    }
    return (long long)g_recs.size();
}

}  // extern "C"
