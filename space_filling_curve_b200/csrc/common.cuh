// common.cuh -- shared helpers of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "tess.h"
#include <utility>

// The pair search that tess_build_neighbors runs when its flags name none
// (TESS_LANE2_SEARCH, TESS_LANE_SEARCH or TESS_TILE_SEARCH): the fastest on
// the 10.24M-atom salt solution as last measured.
#ifndef TESS_DEFAULT_SEARCH
#define TESS_DEFAULT_SEARCH TESS_LANE2_SEARCH
#endif

namespace tess {

constexpr unsigned FULL = 0xffffffffu;

// Number of kernels launched through the library (diagnostic).
extern std::atomic<long long> g_launches;
inline void count_launch(long long k = 1) { g_launches.fetch_add(k, std::memory_order_relaxed); }

// Stage ids for the optional event timing.
enum Stage { ST_KEYS = 0, ST_SORT = 1, ST_CELLS = 2, ST_PAIRS = 3, ST_SKIN = 4, ST_EDGE = 5, ST_BACKWARD = 6, ST_RESORT = 7, ST_MONITOR = 8, ST_COUNT = 9 };

// Records an event pair around a stage when stage timing is enabled; in a
// build with -DTESS_NVTX it also opens an NVTX range named after the stage
// (host-side, around the launches), for timeline profilers.
struct StageScope {
    int stage;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    StageScope(int stage_, cudaStream_t s_);
    ~StageScope();
};

// Stage names, as the Python binding reports them.
inline const char* stage_name(int stage) {
    static const char* const names[ST_COUNT] = {"hilbert_keys", "key_sort", "cell_binning", "pair_search",
                                                "skin_check", "edge_aggregate", "edge_backward", "resort",
                                                "min_pair"};
    return stage >= 0 && stage < ST_COUNT ? names[stage] : "tess";
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a caller-provided workspace.
struct Carve {
    char* base;
    size_t off = 0;
    explicit Carve(void* p) : base(static_cast<char*>(p)) {}
    template <class T>
    T* take(size_t count) {
        off = align_up(off, 256);
        T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
        off += sizeof(T) * count;
        return p;
    }
};

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool finite_pos(float x) { return std::isfinite(x) && x > 0.0f; }

inline tess_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TESS_OK : TESS_ERR_CUDA;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Programmatic dependent launch: kernels of the rebuild path are launched so
// that each may be scheduled while the one before it drains, and each waits
// at its first line (griddepcontrol.wait) until the grids it depends on have
// completed and their memory is visible.  The wait is a no-op for a grid
// launched without the attribute.
#ifndef TESS_PDL
#define TESS_PDL 1
#endif
__device__ __forceinline__ void pdl_wait() {
#if TESS_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

template <typename... P, typename... A>
inline void launch_pdl(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
#if TESS_PDL
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k, std::forward<A>(args)...);
#else
    k<<<grid, block, smem, s>>>(std::forward<A>(args)...);
#endif
}

// Zeroes two ranges of 32-bit words (either may be empty): the resets at
// the start of a call, as a kernel so that the call's chain of launches stays
// programmatic from its first kernel on (a memset would break it).
namespace {
__global__ void zero2_kernel(unsigned* a, size_t na, unsigned* b, size_t nb) {
    pdl_wait();
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < na; k += stride) a[k] = 0u;
    for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < nb; k += stride) b[k] = 0u;
}
}  // namespace
inline void zero2(unsigned* a, size_t na, unsigned* b, size_t nb, int sms, cudaStream_t s) {
    const size_t words = na > nb ? na : nb;
    const unsigned blocks = (unsigned)std::max<size_t>(1, std::min<size_t>((words + 1023) / 1024, (size_t)sms * 4));
    launch_pdl(zero2_kernel, dim3(blocks), dim3(256), 0, s, a, na, b, nb);
    count_launch();
}

// Runs of equal consecutive values among the valid lanes of a warp (the
// valid lanes must be a prefix of the warp, as in a loop over i < n with
// consecutive lanes on consecutive i): the first lane of this lane's run,
// the run's length and this lane's rank in it.  Inputs in curve or cell
// order put equal bins in long runs, so one atomic per run serves as a
// warp-aggregated histogram update; all 32 lanes must call it.
struct WarpRun {
    int leader, len, rank;
};
__device__ __forceinline__ WarpRun warp_run(unsigned v, bool valid) {
    const int lane = threadIdx.x & 31;
    const unsigned prev = __shfl_up_sync(0xffffffffu, v, 1);
    const unsigned heads = __ballot_sync(0xffffffffu, valid && (lane == 0 || v != prev));
    const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));
    const unsigned le = lanemask_lt() | (1u << lane);
    const int leader = 31 - __clz(heads & le);
    const unsigned after = heads & ~le;
    const int end = after ? __ffs(after) - 1 : nvalid;
    return WarpRun{leader, end - leader, lane - leader};
}

// Checked builds (-DTESS_CHECK): an index that a kernel scatters to or
// gathers from is tested against its bound; a bad one sets TESS_DEV_CHECK in
// the status word given and the access is skipped.  In the product build the
// test compiles away.
#ifdef TESS_CHECK
__device__ __forceinline__ bool check_index(long long idx, long long bound, int32_t* status) {
    if (idx >= 0 && idx < bound) return true;
    if (status) atomicOr(status, TESS_DEV_CHECK);
    return false;
}
#else
__device__ __forceinline__ bool check_index(long long, long long, int32_t*) { return true; }
#endif

__device__ __forceinline__ int floor_div(int a, int b) {
    int q = a / b;
    return (a % b != 0 && ((a < 0) != (b < 0))) ? q - 1 : q;
}

}  // namespace tess
