// scan.cuh -- exclusive scan of an int array of any length on the device
// (one launch, decoupled look-back between tiles), used for the cell offsets
// of the neighbor list and the bucket offsets of the sort.  Also the
// look-back word format the radix sort shares.  Internal; each translation
// unit that includes it gets its own copy.
#pragma once

#include "common.cuh"

namespace tess {
namespace {

constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_ITEMS = 4;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_ITEMS;

__device__ __forceinline__ int block_scan_incl(int v, int* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? s_warp[warp - 1] : 0;
    __syncthreads();
    return v + add;
}

// Decoupled look-back state of one tile: a flag in the top two bits (0: not
// yet published), the value below it.
constexpr unsigned long long ST_AGG = 1ull << 62;   // the tile's own total
constexpr unsigned long long ST_INC = 2ull << 62;   // the tile's inclusive prefix
constexpr unsigned long long ST_VAL = (1ull << 62) - 1ull;
constexpr int LOOKBACK_SPIN_LIMIT = 1 << 22;         // polls before a wait gives up

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// One pass: start[c] = cnt[0] + ... + cnt[c - 1] for c <= m.  Each block
// takes the next tile from a counter (so every lower tile has started),
// scans it, publishes its total, then looks back over the lower tiles'
// words -- 32 at a time, one per lane of the last warp -- summing totals
// until it meets an inclusive prefix, and publishes its own.  A wait that
// outlasts LOOKBACK_SPIN_LIMIT polls sets TESS_DEV_TIMEOUT and reads the
// tile as 0, so the kernel always ends.  state: tiles words + 1 (the
// counter), all zero on entry.
__global__ __launch_bounds__(SCAN_THREADS) void scan_lookback_kernel(const int* __restrict__ cnt, long long m,
                                                                     unsigned long long* state,
                                                                     int* __restrict__ start, int32_t* status) {
    __shared__ int s_warp[32];
    __shared__ int s_tile, s_excl;
    pdl_wait();
    const long long tiles = (m + SCAN_TILE - 1) / SCAN_TILE;
    if (threadIdx.x == 0) s_tile = atomicAdd(reinterpret_cast<unsigned*>(state + tiles), 1u);
    __syncthreads();
    const long long t = s_tile;
    const long long b = t * SCAN_TILE + (long long)threadIdx.x * SCAN_ITEMS;
    static_assert(SCAN_ITEMS == 4, "one int4 per thread");
    int v[SCAN_ITEMS];
    if (b + SCAN_ITEMS <= m) {
        const int4 q = *reinterpret_cast<const int4*>(cnt + b);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
        for (int k = 0; k < SCAN_ITEMS; ++k) v[k] = (b + k < m) ? cnt[b + k] : 0;
    }
    const int sum = v[0] + v[1] + v[2] + v[3];
    const int inc = block_scan_incl(sum, s_warp);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == (int)(blockDim.x >> 5) - 1) {
        const int tot = __shfl_sync(FULL, inc, 31);
        if (lane == 0) st_relaxed(state + t, (t == 0 ? ST_INC : ST_AGG) | (unsigned)tot);
        int excl = 0;
        bool timed_out = false;
        for (long long top = t - 1; top >= 0; top -= 32) {
            const long long p = top - lane;
            unsigned long long w = ST_INC;   // below tile 0: an inclusive prefix of 0
            if (p >= 0) {
                int spins = 0;
                while (((w = ld_relaxed(state + p)) & ~ST_VAL) == 0) {
                    if (++spins > LOOKBACK_SPIN_LIMIT) {
                        timed_out = true;
                        w = ST_INC;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            const unsigned incl = __ballot_sync(FULL, (w & ~ST_VAL) == ST_INC);
            const int last = incl ? __ffs(incl) - 1 : 31;   // nearest inclusive word
            excl += __reduce_add_sync(FULL, lane <= last ? (unsigned)(w & ST_VAL) : 0u);
            if (incl) break;
        }
        if (t > 0 && lane == 0) st_relaxed(state + t, ST_INC | (unsigned)(excl + tot));
        if (__any_sync(FULL, timed_out) && lane == 0 && status) atomicOr(status, TESS_DEV_TIMEOUT);
        if (lane == 0) s_excl = excl;
    }
    __syncthreads();
    int run = s_excl + inc - sum;
    int o[SCAN_ITEMS];
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        o[k] = run;
        run += v[k];
    }
    if (b + SCAN_ITEMS <= m) {
        *reinterpret_cast<int4*>(start + b) = make_int4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
        for (int k = 0; k < SCAN_ITEMS; ++k)
            if (b + k < m) start[b + k] = o[k];
    }
    if (b < m && b + SCAN_ITEMS >= m) start[m] = run;   // the thread holding the last element
}

// Words of look-back state exclusive_scan needs for m elements (zero them
// before each call).
inline long long scan_state_len(long long m) { return (m + SCAN_TILE - 1) / SCAN_TILE + 1; }

// start[c] = sum of cnt[0 .. c) for c <= m; cnt and start 16-byte aligned.
inline void exclusive_scan(const int* cnt, long long m, unsigned long long* state, int* start, int32_t* status,
                           cudaStream_t s) {
    const long long tiles = (m + SCAN_TILE - 1) / SCAN_TILE;
    launch_pdl(scan_lookback_kernel, dim3((unsigned)tiles), dim3(SCAN_THREADS), 0, s, cnt, m, state, start, status);
    count_launch();
}

}  // namespace
}  // namespace tess
