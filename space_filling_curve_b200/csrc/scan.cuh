// scan.cuh -- exclusive scan of an int array of any length on the device
// (three launches: per-tile sums, a scan of the sums, per-tile scans), used
// for the cell offsets of the neighbor list and the bucket offsets of the
// sort.  Internal; each translation unit that includes it gets its own copy.
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

// per-tile sums of the counts
__global__ __launch_bounds__(SCAN_THREADS) void scan_reduce_kernel(const int* __restrict__ cnt, long long m,
                                                                   int* __restrict__ sums) {
    __shared__ int s_warp[32];
    pdl_wait();
    const long long b = (long long)blockIdx.x * SCAN_TILE + (long long)threadIdx.x * SCAN_ITEMS;
    int v = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) v += (b + k < m) ? cnt[b + k] : 0;
    const int tot = block_scan_incl(v, s_warp);
    if (threadIdx.x == blockDim.x - 1) sums[blockIdx.x] = tot;
}

// exclusive scan of the per-tile sums, one block, any length
__global__ __launch_bounds__(SCAN_THREADS) void scan_sums_kernel(int* sums, long long nt) {
    __shared__ int s_warp[32];
    pdl_wait();
    __shared__ int s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (long long b = 0; b < nt; b += SCAN_THREADS) {
        const long long k = b + threadIdx.x;
        const int v = k < nt ? sums[k] : 0;
        const int inc = block_scan_incl(v, s_warp);
        const int carry = s_carry;
        if (k < nt) sums[k] = carry + inc - v;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) s_carry = carry + inc;
        __syncthreads();
    }
}

// cell_start[c] = exclusive prefix; cnt[c] reset to 0 for the scatter cursor
__global__ __launch_bounds__(SCAN_THREADS) void scan_apply_kernel(int* __restrict__ cnt, long long m,
                                                                  const int* __restrict__ sums,
                                                                  int* __restrict__ cell_start) {
    __shared__ int s_warp[32];
    pdl_wait();
    const long long b = (long long)blockIdx.x * SCAN_TILE + (long long)threadIdx.x * SCAN_ITEMS;
    int v[SCAN_ITEMS];
    int tot = 0;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        v[k] = (b + k < m) ? cnt[b + k] : 0;
        tot += v[k];
    }
    const int inc = block_scan_incl(tot, s_warp);
    int run = sums[blockIdx.x] + inc - tot;
#pragma unroll
    for (int k = 0; k < SCAN_ITEMS; ++k) {
        if (b + k < m) {
            cell_start[b + k] = run;
            cnt[b + k] = 0;
        }
        run += v[k];
    }
    if (b < m && b + SCAN_ITEMS >= m) cell_start[m] = run;   // the thread holding the last cell
}


// Launches the three kernels: start[c] = sum of cnt[0 .. c) for c <= m, and
// cnt is reset to 0 (a scatter cursor).  sums holds scan_sums_len(m) ints.
inline long long scan_sums_len(long long m) { return (m + SCAN_TILE - 1) / SCAN_TILE + 1; }
inline void exclusive_scan(int* cnt, long long m, int* sums, int* start, cudaStream_t s) {
    const long long tiles = (m + SCAN_TILE - 1) / SCAN_TILE;
    launch_pdl(scan_reduce_kernel, dim3((unsigned)tiles), dim3(SCAN_THREADS), 0, s, (const int*)cnt, m, sums);
    launch_pdl(scan_sums_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, sums, tiles);
    launch_pdl(scan_apply_kernel, dim3((unsigned)tiles), dim3(SCAN_THREADS), 0, s, cnt, m, (const int*)sums, start);
    count_launch(3);
}

}  // namespace
}  // namespace tess
