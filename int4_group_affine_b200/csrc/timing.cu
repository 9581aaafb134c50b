// timing.cu - opt-in CUDA-event timing of the library's kernel launches.
#include <vector>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kMaxRecords = 1 << 16;

const char* const kNames[kKindCount] = {
    "pack", "dequant", "router_logits", "topk", "index_count", "index_scan", "index_scatter",
    "lora_a", "gate_up", "down", "combine", "rmsnorm", "mixed_gate_up", "mixed_down", "mixed_linear",
    "decode_fused", "tc_lora_gate_up", "tc_gate_up", "tc_lora_down", "tc_down", "tc_router", "kperm", "decode_chain", "prerouter", "act8", "mixed_a8", "ep_dispatch", "ep_combine", "decode_cluster",
};

struct Rec {
    int kind;  // -1: start marker of an entry point
};

bool g_enabled = false;
std::vector<cudaEvent_t> g_pool;
std::vector<Rec> g_recs;

void record(int kind, cudaStream_t s) {
    if (!g_enabled || (int)g_recs.size() >= kMaxRecords) return;
    const size_t i = g_recs.size();
    if (i >= g_pool.size()) {
        cudaEvent_t ev;
        if (cudaEventCreate(&ev) != cudaSuccess) return;
        g_pool.push_back(ev);
    }
    // Under stream capture the record becomes an event node of the graph, so the
    // times come from the graph's replay.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return;
    const cudaError_t e = cap == cudaStreamCaptureStatusActive
                              ? cudaEventRecordWithFlags(g_pool[i], s, cudaEventRecordExternal)
                              : cudaEventRecord(g_pool[i], s);
    if (e != cudaSuccess) return;
    g_recs.push_back(Rec{kind});
}

}  // namespace

// Start of an entry point's launch sequence.  Also drops a stale, non-sticky
// error left by an earlier runtime call, so that the launch checks that follow
// report this call's launches only (sticky device errors persist regardless).
void timing_begin(cudaStream_t s) {
    (void)cudaGetLastError();
    record(-1, s);
}
void timing_mark(int kind, cudaStream_t s) { record(kind, s); }

}  // namespace moeq

using namespace moeq;

extern "C" {

int moe_timing_kinds(void) { return kKindCount; }

const char* moe_timing_kind_name(int kind) { return (kind >= 0 && kind < kKindCount) ? kNames[kind] : "?"; }

moe_status moe_timing_enable(int enable) {
    g_enabled = enable != 0;
    if (!g_enabled) g_recs.clear();
    return MOE_OK;
}

moe_status moe_timing_collect(float* total_ms, int32_t* launches, int32_t n_kinds) {
    if (!total_ms || !launches || n_kinds < 0) return MOE_ERR_INVALID_ARG;
    if (!g_recs.empty() && cudaEventSynchronize(g_pool[g_recs.size() - 1]) != cudaSuccess) {
        g_recs.clear();
        return MOE_ERR_CUDA;
    }
    bool missing = false;
    for (size_t i = 1; i < g_recs.size(); ++i) {
        const int k = g_recs[i].kind;
        if (k < 0 || k >= n_kinds) continue;
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, g_pool[i - 1], g_pool[i]) != cudaSuccess) {
            missing = true;  // e.g. events of a captured graph that was not replayed
            continue;
        }
        total_ms[k] += ms;
        launches[k] += 1;
    }
    g_recs.clear();
    if (missing) (void)cudaGetLastError();  // do not leave the query's error for the next launch check
    return MOE_OK;
}

}  // extern "C"
