// scan.cuh -- exclusive scan of an int array of any length on the device
// (one launch, decoupled look-back between chunks), used for the cell offsets
// of the neighbor list and the bucket offsets of the sort.  Also the
// look-back word format the radix sort shares.  Internal; each translation
// unit that includes it gets its own copy.
#pragma once

#include "common.cuh"

namespace tess {
namespace {

constexpr int SCAN_THREADS = 512;
constexpr int SCAN_SUB = SCAN_THREADS * 4;     // elements per block step (one int4 per thread)
constexpr int SCAN_MAX_CHUNKS = 1024;          // blocks of one scan at most

// Inclusive scan of one value per thread over the block; *tot = block total.
__device__ __forceinline__ int block_scan_incl(int v, int* s_warp, int* tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (int)(blockDim.x >> 5);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < nw) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? s_warp[warp - 1] : 0;
    *tot = s_warp[nw - 1];
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

// One launch: start[c] = cnt[0] + ... + cnt[c - 1] for c <= m.  The array
// is cut into chunks, one per block, taken in order from a counter (so every
// lower chunk's block has started).  A block sums its chunk, publishes the
// total, looks back over the lower chunks' words -- 32 at a time, one per
// lane of warp 0 -- summing totals until it meets an inclusive prefix,
// publishes its own, then scans its chunk (a second read, from L2).  A wait
// that outlasts LOOKBACK_SPIN_LIMIT polls sets TESS_DEV_TIMEOUT and reads
// the chunk as 0, so the kernel always ends.  state: nchunks words + 1 (the
// counter), all zero on entry; chunk a multiple of 4.
__global__ __launch_bounds__(SCAN_THREADS) void scan_lookback_kernel(const int* __restrict__ cnt, long long m,
                                                                     long long chunk, int nchunks,
                                                                     unsigned long long* state,
                                                                     int* __restrict__ start, int32_t* status) {
    __shared__ int s_warp[32];
    __shared__ int s_tile, s_excl;
    pdl_wait();
    if (threadIdx.x == 0) s_tile = atomicAdd(reinterpret_cast<unsigned*>(state + nchunks), 1u);
    __syncthreads();
    const int t = s_tile;
    const long long beg = (long long)t * chunk, end = beg + chunk < m ? beg + chunk : m;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    int sum = 0;
    for (long long b = beg + 4 * (long long)threadIdx.x; b < end; b += SCAN_SUB) {
        if (b + 4 <= end) {
            const int4 q = *reinterpret_cast<const int4*>(cnt + b);
            sum += q.x + q.y + q.z + q.w;
        } else {
            for (long long k = b; k < end; ++k) sum += cnt[k];
        }
    }
    sum = (int)__reduce_add_sync(FULL, (unsigned)sum);
    if (lane == 0) s_warp[warp] = sum;
    __syncthreads();
    if (warp == 0) {
        const int tot = (int)__reduce_add_sync(FULL, lane < (int)(blockDim.x >> 5) ? (unsigned)s_warp[lane] : 0u);
        if (lane == 0) st_relaxed(state + t, (t == 0 ? ST_INC : ST_AGG) | (unsigned)tot);
        int excl = 0;
        bool timed_out = false;
        for (long long top = (long long)t - 1; top >= 0; top -= 32) {
            const long long p = top - lane;
            unsigned long long w = ST_INC;   // below chunk 0: an inclusive prefix of 0
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
            excl += (int)__reduce_add_sync(FULL, lane <= last ? (unsigned)(w & ST_VAL) : 0u);
            if (incl) break;
        }
        if (t > 0 && lane == 0) st_relaxed(state + t, ST_INC | (unsigned)(excl + tot));
        if (__any_sync(FULL, timed_out) && lane == 0 && status) atomicOr(status, TESS_DEV_TIMEOUT);
        if (lane == 0) s_excl = excl;
    }
    __syncthreads();

    int carry = s_excl;
    for (long long b0 = beg; b0 < end; b0 += SCAN_SUB) {
        const long long b = b0 + 4 * (long long)threadIdx.x;
        int v[4] = {0, 0, 0, 0};
        if (b + 4 <= end) {
            const int4 q = *reinterpret_cast<const int4*>(cnt + b);
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = (b + k < end) ? cnt[b + k] : 0;
        }
        const int own = v[0] + v[1] + v[2] + v[3];
        int tot;
        const int inc = block_scan_incl(own, s_warp, &tot);
        int o[4];
        int run = carry + inc - own;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            o[k] = run;
            run += v[k];
        }
        if (b + 4 <= end) {
            *reinterpret_cast<int4*>(start + b) = make_int4(o[0], o[1], o[2], o[3]);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (b + k < end) start[b + k] = o[k];
        }
        if (b < m && b + 4 >= m) start[m] = run;   // the thread holding the last element
        carry += tot;
    }
    if (m == 0 && threadIdx.x == 0) start[0] = 0;
}

// Chunks of a scan of m elements on sms SMs (a multiple of 4 elements each).
struct ScanPlan {
    long long chunk;
    int nchunks;
};
inline ScanPlan scan_plan(long long m, int sms) {
    const long long subs = (m + SCAN_SUB - 1) / SCAN_SUB;
    const long long want = std::max<long long>(1, std::min<long long>(subs, std::min(sms * 4, SCAN_MAX_CHUNKS)));
    long long chunk = (m + want - 1) / want;
    chunk = std::max<long long>(4, (chunk + 3) / 4 * 4);
    return ScanPlan{chunk, (int)std::max<long long>(1, (m + chunk - 1) / chunk)};
}

// Words of look-back state exclusive_scan needs for m elements (zero them
// before each call).
inline long long scan_state_len(long long m) {
    return std::max<long long>(1, std::min<long long>((m + SCAN_SUB - 1) / SCAN_SUB, SCAN_MAX_CHUNKS)) + 1;
}

// start[c] = sum of cnt[0 .. c) for c <= m; cnt and start 16-byte aligned.
inline void exclusive_scan(const int* cnt, long long m, unsigned long long* state, int* start, int32_t* status,
                           int sms, cudaStream_t s) {
    const ScanPlan P = scan_plan(m, sms);
    launch_pdl(scan_lookback_kernel, dim3((unsigned)P.nchunks), dim3(SCAN_THREADS), 0, s, cnt, m, P.chunk,
               P.nchunks, state, start, status);
    count_launch();
}

}  // namespace
}  // namespace tess
