// capi.cu -- the extern "C" boundary of libtess.so (declared in tess.h).
#include <mutex>
#include <vector>

#include "common.cuh"

#ifdef TESS_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace tess {

std::atomic<long long> g_launches{0};

size_t hilbert_sort_workspace(int n);
size_t hilbert_resort_workspace(int n);
size_t lookback_probe_workspace();
tess_status lookback_timeout_probe(void* ws, size_t ws_bytes, int32_t* status, cudaStream_t s);
size_t min_pair_workspace();
tess_status min_pair_distance(const float* pos, int n, tess_box box, const int32_t* nbr, const int32_t* counts,
                              int cap, void* ws, size_t ws_bytes, double* min_r2, int32_t* min_pair,
                              cudaStream_t s);
tess_status hilbert_resort(const float* pos, int n, tess_box box, int bits, const int32_t* perm_prev,
                           const uint32_t* keys_prev, void* ws, size_t ws_bytes, int32_t* perm,
                           uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s);
tess_status hilbert_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                         uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s);
tess_status morton_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                        uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s);
size_t build_neighbors_workspace(int n, tess_box box, float rc, float skin);
tess_status build_neighbors(const float* pos, int n, tess_box box, float rc, float skin, int cap, int flags,
                            void* ws, size_t ws_bytes, int32_t* nbr, int32_t* counts, int32_t* overflow,
                            cudaStream_t s);
tess_status skin_check(const float* pos, const float* pos_ref, int n, tess_box box, float skin, int32_t* rebuild,
                       double* max_disp2, cudaStream_t s);
tess_status edge_aggregate(const float* pos, int n, tess_box box, float rc, const int32_t* nbr, const int32_t* counts,
                           int cap, const float* feat, int F, float* out, float* edge_vec, float* edge_fc,
                           float* edge_unit, cudaStream_t s);

tess_status edge_backward(const float* pos, int n, tess_box box, float rc, const int32_t* nbr, const int32_t* counts,
                          int cap, const float* feat, const float* grad_out, int F, float* grad_feat,
                          float* grad_pos, cudaStream_t s);

// ---------------------------------------------------------------- stage timing

namespace {
// Stage timing state.  Events are recycled through a pool: a scope takes two
// from the pool (creating them only when it is empty) and tess_stage_times
// gives them back, so a warmed-up timing loop creates no events.
struct Timing {
    std::mutex mu;
    bool enabled = false;
    struct Rec {
        int stage;
        cudaEvent_t a, b;
    };
    std::vector<Rec> recs;
    std::vector<cudaEvent_t> pool;
    cudaEvent_t take() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return e;
    }
};
Timing& timing() {
    static Timing t;
    return t;
}
}  // namespace

StageScope::StageScope(int stage_, cudaStream_t s_) : stage(stage_), s(s_) {
#ifdef TESS_NVTX
    nvtxRangePushA(stage_name(stage));
#endif
    Timing& t = timing();
    std::lock_guard<std::mutex> g(t.mu);
    if (!t.enabled) return;
    // no timing inside a graph capture: event nodes are not allowed in every
    // graph (conditional bodies), and a captured stage runs at replay time
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
    a = t.take();
    b = t.take();
    if (!a || !b) {
        if (a) t.pool.push_back(a);
        if (b) t.pool.push_back(b);
        a = b = nullptr;
        return;
    }
    cudaEventRecord(a, s);
}

StageScope::~StageScope() {
#ifdef TESS_NVTX
    nvtxRangePop();
#endif
    if (!a) return;
    cudaEventRecord(b, s);
    Timing& t = timing();
    std::lock_guard<std::mutex> g(t.mu);
    t.recs.push_back({stage, a, b});
}

}  // namespace tess

using namespace tess;

extern "C" {

const char* tess_status_string(tess_status s) {
    switch (s) {
        case TESS_OK: return "ok";
        case TESS_ERR_INVALID_ARG: return "invalid argument";
        case TESS_ERR_BOX_TOO_SMALL: return "box too small: some length below twice the cutoff radius";
        case TESS_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case TESS_ERR_CUDA: return "CUDA launch error";
        case TESS_ERR_TOO_LARGE: return "n above the capacity of the static scratch (TESS_HILBERT_SORT_STATIC_MAX_N)";
    }
    return "unknown status";
}

const char* tess_version(void) {
    return TESS_DEFAULT_SEARCH == TESS_LANE2_SEARCH ? "tess-b200 0.3 (sm_100a; default pair search: two atoms per lane)"
           : TESS_DEFAULT_SEARCH == TESS_LANE_SEARCH ? "tess-b200 0.3 (sm_100a; default pair search: per-lane)"
                                                     : "tess-b200 0.3 (sm_100a; default pair search: tile)";
}

long long tess_kernel_launch_count(void) { return g_launches.load(); }

size_t tess_hilbert_sort_workspace(int n) { return hilbert_sort_workspace(n); }

tess_status tess_hilbert_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes,
                              int32_t* perm, uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status,
                              tess_stream_t stream) {
    return hilbert_sort(pos, n, box, bits, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t tess_hilbert_resort_workspace(int n) { return hilbert_resort_workspace(n); }

size_t tess_debug_lookback_timeout_workspace(void) { return lookback_probe_workspace(); }

tess_status tess_debug_lookback_timeout(void* ws, size_t ws_bytes, int32_t* dev_status, tess_stream_t stream) {
    return lookback_timeout_probe(ws, ws_bytes, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

size_t tess_min_pair_distance_workspace(void) { return min_pair_workspace(); }

tess_status tess_min_pair_distance(const float* pos, int n, tess_box box, const int32_t* nbr,
                                   const int32_t* counts, int max_neighbors, void* ws, size_t ws_bytes,
                                   double* min_r2, int32_t* min_pair, tess_stream_t stream) {
    return min_pair_distance(pos, n, box, nbr, counts, max_neighbors, ws, ws_bytes, min_r2, min_pair,
                             reinterpret_cast<cudaStream_t>(stream));
}

tess_status tess_hilbert_resort(const float* pos, int n, tess_box box, int bits, const int32_t* perm_prev,
                                const uint32_t* keys_prev, void* ws, size_t ws_bytes, int32_t* perm,
                                uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status,
                                tess_stream_t stream) {
    return hilbert_resort(pos, n, box, bits, perm_prev, keys_prev, ws, ws_bytes, perm, keys_sorted, pos_sorted,
                          dev_status, reinterpret_cast<cudaStream_t>(stream));
}

tess_status tess_morton_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes,
                             int32_t* perm, uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status,
                             tess_stream_t stream) {
    return morton_sort(pos, n, box, bits, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t tess_build_neighbors_workspace(int n, tess_box box, float rc, float skin) {
    return build_neighbors_workspace(n, box, rc, skin);
}

tess_status tess_build_neighbors(const float* pos, int n, tess_box box, float rc, float skin, int max_neighbors,
                                 int flags, void* ws, size_t ws_bytes, int32_t* nbr, int32_t* counts,
                                 int32_t* overflow, tess_stream_t stream) {
    return build_neighbors(pos, n, box, rc, skin, max_neighbors, flags, ws, ws_bytes, nbr, counts, overflow,
                           reinterpret_cast<cudaStream_t>(stream));
}

tess_status tess_skin_check(const float* pos, const float* pos_ref, int n, tess_box box, float skin,
                            int32_t* rebuild, double* max_disp2, tess_stream_t stream) {
    return skin_check(pos, pos_ref, n, box, skin, rebuild, max_disp2, reinterpret_cast<cudaStream_t>(stream));
}

tess_status tess_edge_aggregate(const float* pos, int n, tess_box box, float rc, const int32_t* nbr,
                                const int32_t* counts, int max_neighbors, const float* feat, int F, float* out,
                                float* edge_vec, float* edge_fc, float* edge_unit, tess_stream_t stream) {
    return edge_aggregate(pos, n, box, rc, nbr, counts, max_neighbors, feat, F, out, edge_vec, edge_fc, edge_unit,
                          reinterpret_cast<cudaStream_t>(stream));
}

tess_status tess_edge_aggregate_backward(const float* pos, int n, tess_box box, float rc, const int32_t* nbr,
                                         const int32_t* counts, int max_neighbors, const float* feat,
                                         const float* grad_out, int F, float* grad_feat, float* grad_pos,
                                         tess_stream_t stream) {
    return edge_backward(pos, n, box, rc, nbr, counts, max_neighbors, feat, grad_out, F, grad_feat, grad_pos,
                         reinterpret_cast<cudaStream_t>(stream));
}

void tess_stage_timing(int enable) {
    Timing& t = timing();
    std::lock_guard<std::mutex> g(t.mu);
    t.enabled = enable != 0;
}

int tess_stage_times(double* ms_out, long long* calls_out, int max_stages) {
    Timing& t = timing();
    std::vector<Timing::Rec> recs;
    {
        std::lock_guard<std::mutex> g(t.mu);
        recs.swap(t.recs);
    }
    const int ns = std::min<int>(max_stages, ST_COUNT);
    for (int k = 0; k < ns; ++k) {
        ms_out[k] = 0.0;
        if (calls_out) calls_out[k] = 0;
    }
    for (auto& r : recs) {
        float ms = 0.f;
        cudaEventSynchronize(r.b);
        if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess && r.stage < ns) {
            ms_out[r.stage] += ms;
            if (calls_out) calls_out[r.stage] += 1;
        }
    }
    cudaGetLastError();
    {
        std::lock_guard<std::mutex> g(t.mu);
        for (auto& r : recs) {
            t.pool.push_back(r.a);
            t.pool.push_back(r.b);
        }
    }
    return ns;
}

}  // extern "C"
