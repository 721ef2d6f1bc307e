// static_scratch.cu -- tess_hilbert_sort_static: the Hilbert sort for callers
// that cannot allocate device memory.
//
// Some programs that would use this library do not own their device memory:
// an MD engine that loads the neighbor pipeline as a plugin and hands it only
// the position and output buffers it allocated itself, or a time-step loop
// that must never call cudaMalloc (which synchronises the whole device) and
// has no spare buffer to lend as a workspace.  For them this entry point runs
// the same sort kernels on a scratch area that the library carries itself: a
// fixed array in device memory, sized for TESS_HILBERT_SORT_STATIC_MAX_N atoms
// (TESS_HILBERT_SORT_STATIC_BYTES, 21 MiB).  Every GPU that loads the library holds that array until
// the process exits.
//
// The array is shared by every call on a device and keeps what the previous
// call left in it; the sort clears the parts that must start at zero (digit
// histograms, tile counters, look-back states) at the start of each call.
// Two calls whose kernels overlap on the GPU -- on different streams, or from
// different host threads without ordering -- race on the array and corrupt
// each other's results: order them on one stream.
#include "common.cuh"

namespace tess {

size_t hilbert_sort_workspace(int n);
tess_status hilbert_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                         uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s);

constexpr size_t STATIC_SORT_SCRATCH_BYTES = TESS_HILBERT_SORT_STATIC_BYTES;

// The scratch area.  Host code must not pass the name itself to a kernel (on
// the host it is a stand-in, not a device address); its device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_sort_scratch[STATIC_SORT_SCRATCH_BYTES];

namespace {
// Device address of the scratch array in the current context.  It is looked
// up on every call (a host-side query that enqueues no work) rather than
// cached: a cached address would go stale once the context that holds the
// module is destroyed and created again (cudaDeviceReset, or the primary
// context released and retained), and the next call would then write
// through it.
tess_status scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_sort_scratch);
    if (e != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return TESS_ERR_CUDA;
    }
    *out = p;
    return TESS_OK;
}
}  // namespace

}  // namespace tess

extern "C" tess_status tess_hilbert_sort_static(const float* pos, int n, tess_box box, int bits, int32_t* perm,
                                                uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status,
                                                tess_stream_t stream) {
    using namespace tess;
    if (n > TESS_HILBERT_SORT_STATIC_MAX_N) return TESS_ERR_TOO_LARGE;
    if (n <= 0) return TESS_ERR_INVALID_ARG;
    if (hilbert_sort_workspace(n) > STATIC_SORT_SCRATCH_BYTES) return TESS_ERR_TOO_LARGE;
    void* ws = nullptr;
    const tess_status st = scratch_address(&ws);
    if (st != TESS_OK) return st;
    return hilbert_sort(pos, n, box, bits, ws, STATIC_SORT_SCRATCH_BYTES, perm, keys_sorted, pos_sorted, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}
