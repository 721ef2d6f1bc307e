// step_graph.cu -- one time step of the path as a CUDA graph whose rebuild
// branch is taken on the device: Tessera replays each interval between
// rebuilds as one CUDA graph (Tessera, abstract); here the skin check's flag
// drives a conditional node, so a whole MD loop runs with no host round trip
// per step, rebuilds included.
//
//   gather_sorted      current positions into the sorted order of the last rebuild
//   skin_check         max displacement since the last rebuild -> flag
//   step_set_cond      flag (or a pending forced rebuild) -> the IF node's condition
//   IF: hilbert_sort, build_neighbors, pos_cur = pos_sorted
//   edge_aggregate     over the list, at the current positions
#include <vector>

#include "common.cuh"

namespace tess {

tess_status hilbert_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                         uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s);
tess_status build_neighbors(const float* pos, int n, tess_box box, float rc, float skin, int max_neighbors,
                            int flags, void* ws, size_t ws_bytes, int32_t* nbr, int32_t* counts, int32_t* overflow,
                            cudaStream_t s);
size_t hilbert_sort_workspace(int n);
size_t build_neighbors_workspace(int n, tess_box box, float rc, float skin);
tess_status skin_check(const float* pos, const float* pos_ref, int n, tess_box box, float skin, int32_t* rebuild,
                       double* max_disp2, cudaStream_t s);
tess_status edge_aggregate(const float* pos, int n, tess_box box, float rc, const int32_t* nbr, const int32_t* counts,
                           int cap, const float* feat, int F, float* out, float* edge_vec, float* edge_fc,
                           float* edge_unit, cudaStream_t s);

// pos_cur[k] = (pos[perm[k]], 0); an index outside [0, n) (perm not yet
// written) gives 0, so the first step reads only valid memory.
__global__ __launch_bounds__(256) void gather_sorted_kernel(const float* __restrict__ pos,
                                                            const int32_t* __restrict__ perm, int n,
                                                            float4* __restrict__ pos_cur) {
    for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (long long)gridDim.x * blockDim.x) {
        const int j = perm[k];
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j >= 0 && j < n) v = make_float4(pos[3 * (size_t)j], pos[3 * (size_t)j + 1], pos[3 * (size_t)j + 2], 0.f);
        pos_cur[k] = v;
    }
}

// The step's decision: rebuild when the skin check says so or a rebuild was
// requested (control[0], cleared here); control[1] counts rebuilds.
__global__ void step_set_cond(cudaGraphConditionalHandle h, int32_t* rebuild, int32_t* control) {
    const int r = (*rebuild != 0 || control[0] != 0) ? 1 : 0;
    control[0] = 0;
    control[1] += r;
    *rebuild = r;
    cudaGraphSetConditional(h, (unsigned)r);
}

__global__ void step_request_rebuild(int32_t* control, int reset_count) {
    control[0] = 1;
    if (reset_count) control[1] = 0;
}

}  // namespace tess

struct tess_step_graph {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
};

using namespace tess;

namespace {

// Ends a capture left open by an error and drops what it captured.
void abort_capture(cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone) {
        cudaGraph_t g = nullptr;
        cudaStreamEndCapture(s, &g);
    }
    cudaGetLastError();
}

tess_status check_buffers(const tess_step_buffers* b) {
    if (!b || b->n <= 0 || !b->pos || !b->feat || !b->ws_sort || !b->ws_list || !b->perm || !b->keys ||
        !b->pos_sorted || !b->pos_cur || !b->nbr || !b->counts || !b->overflow || !b->sort_status || !b->rebuild ||
        !b->max_disp2 || !b->control || !b->out || b->max_neighbors < 1 || b->F < 1 || b->bits < 1 || b->bits > 10)
        return TESS_ERR_INVALID_ARG;
    if (!(b->rc > 0.f) || !(b->skin >= 0.f) || !finite_pos(b->box.lx) || !finite_pos(b->box.ly) ||
        !finite_pos(b->box.lz))
        return TESS_ERR_INVALID_ARG;
    if (b->ws_sort_bytes < hilbert_sort_workspace(b->n) ||
        b->ws_list_bytes < build_neighbors_workspace(b->n, b->box, b->rc, b->skin))
        return TESS_ERR_WORKSPACE_TOO_SMALL;
    return TESS_OK;
}

}  // namespace

extern "C" {

tess_status tess_step_graph_create(const tess_step_buffers* b, tess_stream_t stream, tess_step_graph** out) {
    if (!out) return TESS_ERR_INVALID_ARG;
    *out = nullptr;
    tess_status st = check_buffers(b);
    if (st != TESS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!s) return TESS_ERR_INVALID_ARG;     // capture needs a stream other than the legacy default
    const cudaStreamCaptureMode mode = cudaStreamCaptureModeThreadLocal;
    tess_step_graph* G = new tess_step_graph();
    auto fail = [&](tess_status code) {
        abort_capture(s);
        if (G->exec) cudaGraphExecDestroy(G->exec);
        if (G->graph) cudaGraphDestroy(G->graph);
        delete G;
        return code;
    };
    if (cudaGraphCreate(&G->graph, 0) != cudaSuccess) return fail(TESS_ERR_CUDA);
    cudaGraphConditionalHandle h;
    if (cudaGraphConditionalHandleCreate(&h, G->graph, 0, 0) != cudaSuccess) return fail(TESS_ERR_CUDA);

    // part 1: gather, skin check, decision
    if (cudaStreamBeginCaptureToGraph(s, G->graph, nullptr, nullptr, 0, mode) != cudaSuccess) return fail(TESS_ERR_CUDA);
    {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int blocks = (int)std::min<long long>(((long long)b->n + 255) / 256, (long long)sms * 8);
        gather_sorted_kernel<<<blocks, 256, 0, s>>>(b->pos, b->perm, b->n, reinterpret_cast<float4*>(b->pos_cur));
        count_launch();
    }
    st = skin_check(b->pos_cur, b->pos_sorted, b->n, b->box, b->skin, b->rebuild, b->max_disp2, s);
    if (st != TESS_OK) return fail(st);
    step_set_cond<<<1, 1, 0, s>>>(h, b->rebuild, b->control);
    count_launch();
    std::vector<cudaGraphNode_t> deps;
    {
        cudaStreamCaptureStatus cs;
        const cudaGraphNode_t* d = nullptr;
        size_t nd = 0;
        if (cudaStreamGetCaptureInfo(s, &cs, nullptr, nullptr, &d, &nd) != cudaSuccess) return fail(TESS_ERR_CUDA);
        deps.assign(d, d + nd);
    }
    if (cudaStreamEndCapture(s, &G->graph) != cudaSuccess) return fail(TESS_ERR_CUDA);

    // part 2: the rebuild branch
    cudaGraphNodeParams p = {};
    p.type = cudaGraphNodeTypeConditional;
    p.conditional.handle = h;
    p.conditional.type = cudaGraphCondTypeIf;
    p.conditional.size = 1;
    cudaGraphNode_t cond_node;
    if (cudaGraphAddNode(&cond_node, G->graph, deps.data(), deps.size(), &p) != cudaSuccess) return fail(TESS_ERR_CUDA);
    cudaGraph_t body = p.conditional.phGraph_out[0];
    if (cudaStreamBeginCaptureToGraph(s, body, nullptr, nullptr, 0, mode) != cudaSuccess) return fail(TESS_ERR_CUDA);
    st = hilbert_sort(b->pos, b->n, b->box, b->bits, b->ws_sort, b->ws_sort_bytes, b->perm, b->keys, b->pos_sorted,
                      b->sort_status, s);
    if (st != TESS_OK) return fail(st);
    st = build_neighbors(b->pos_sorted, b->n, b->box, b->rc, b->skin, b->max_neighbors, b->flags, b->ws_list,
                         b->ws_list_bytes, b->nbr, b->counts, b->overflow, s);
    if (st != TESS_OK) return fail(st);
    if (cudaMemcpyAsync(b->pos_cur, b->pos_sorted, (size_t)b->n * sizeof(float4), cudaMemcpyDeviceToDevice, s) !=
        cudaSuccess)
        return fail(TESS_ERR_CUDA);
    if (cudaStreamEndCapture(s, &body) != cudaSuccess) return fail(TESS_ERR_CUDA);

    // part 3: the aggregation after the branch
    if (cudaStreamBeginCaptureToGraph(s, G->graph, &cond_node, nullptr, 1, mode) != cudaSuccess)
        return fail(TESS_ERR_CUDA);
    st = edge_aggregate(b->pos_cur, b->n, b->box, b->rc, b->nbr, b->counts, b->max_neighbors, b->feat, b->F, b->out,
                        nullptr, nullptr, nullptr, s);
    if (st != TESS_OK) return fail(st);
    if (cudaStreamEndCapture(s, &G->graph) != cudaSuccess) return fail(TESS_ERR_CUDA);

    if (cudaGraphInstantiate(&G->exec, G->graph, 0) != cudaSuccess) return fail(TESS_ERR_CUDA);
    // the first launch builds the list
    step_request_rebuild<<<1, 1, 0, s>>>(b->control, 1);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return fail(TESS_ERR_CUDA);
    *out = G;
    return TESS_OK;
}

tess_status tess_step_graph_launch(tess_step_graph* g, tess_stream_t stream) {
    if (!g || !g->exec) return TESS_ERR_INVALID_ARG;
    return cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? TESS_OK : TESS_ERR_CUDA;
}

tess_status tess_step_graph_request_rebuild(const tess_step_buffers* b, tess_stream_t stream) {
    if (!b || !b->control) return TESS_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    step_request_rebuild<<<1, 1, 0, s>>>(b->control, 0);
    count_launch();
    return launch_status();
}

void tess_step_graph_destroy(tess_step_graph* g) {
    if (!g) return;
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    delete g;
}

}  // extern "C"
