// hilbert_sort.cu -- Hilbert keys and the device radix sort that orders atoms
// along the curve (Tessera orders atoms along a space-filling curve; Tessera,
// abstract).
//
// Pipeline (one stream, no host sync):
//   keys_kernel      positions -> 64-bit elements (key << 32 | index), plus
//                    the digit histograms of every radix pass
//   onesweep_pass    one stable LSD pass per 8-bit digit: tile-local ranking
//                    with warp match, decoupled look-back across tiles for
//                    the global digit offsets, coalesced scatter from a
//                    digit-sorted shared-memory copy of the tile.  The last
//                    pass writes perm / keys / float4 positions directly.
// Elements carry the input index in the low word, so equal keys keep input
// order (stable passes) and the permutation is unique.
#include <algorithm>

#include "common.cuh"
#include "hilbert_table.cuh"
#include "scan.cuh"

namespace tess {

// ---------------------------------------------------------------- keys

// Spread the low 10 bits of v so that bit k lands on bit 3k.
__device__ __forceinline__ uint32_t spread3(uint32_t v) {
    v &= 0x3ffu;
    v = (v | (v << 16)) & 0x030000ffu;
    v = (v | (v << 8)) & 0x0300f00fu;
    v = (v | (v << 4)) & 0x030c30c3u;
    v = (v | (v << 2)) & 0x09249249u;
    return v;
}

// Grid cell of one coordinate: floor(x * scale) with one fp32 multiply,
// clamped into [0, top]; products below 1 (negative, NaN) give 0.
__device__ __forceinline__ uint32_t quantize(float x, float scale, uint32_t top) {
    float prod = __fmul_rn(x, scale);
    if (!(prod >= 1.0f)) return 0u;
    float fl = floorf(prod);
    return fl >= (float)top ? top : (uint32_t)fl;
}

// The same index from the Morton code m of the point by the state machine of
// hilbert_table.cuh: one shared-memory lookup per two levels (and one for
// the top level when bits is odd).
constexpr int HT_STATES = kHilbertTables.nstates;
struct alignas(16) HilbertSmem {
    uint16_t two[HT_STATES * 64];
    uint16_t one[HT_STATES * 8];
};
static_assert(sizeof(HilbertSmem) % 4 == 0, "copied as words");
__device__ const HilbertTables d_hilbert_tables = kHilbertTables;

__device__ __forceinline__ void load_hilbert_tables(HilbertSmem& S) {
    const uint32_t* two = reinterpret_cast<const uint32_t*>(d_hilbert_tables.two);
    const uint32_t* one = reinterpret_cast<const uint32_t*>(d_hilbert_tables.one);
    uint32_t* d2 = reinterpret_cast<uint32_t*>(S.two);
    uint32_t* d1 = reinterpret_cast<uint32_t*>(S.one);
    for (int k = threadIdx.x; k < HT_STATES * 32; k += blockDim.x) d2[k] = two[k];
    for (int k = threadIdx.x; k < HT_STATES * 4; k += blockDim.x) d1[k] = one[k];
}

__device__ __forceinline__ uint32_t hilbert_key_fsm(uint32_t m, int bits, const HilbertSmem& S) {
    uint32_t st = 0u, key = 0u;
    int l = bits;
    if (l & 1) {
        const uint32_t e = S.one[(m >> (3 * (l - 1))) & 7u];
        key = e & 7u;
        st = e >> 6;
        --l;
    }
    for (; l > 0; l -= 2) {
        const uint32_t e = S.two[(st << 6) | ((m >> (3 * (l - 2))) & 63u)];
        key = (key << 6) | (e & 63u);
        st = e >> 6;
    }
    return key;
}

constexpr int KEYS_THREADS = 256;
constexpr int RADIX = 256;
constexpr int MAX_PASSES = 4;

// Morton (Z-order) index: the three words interleaved with no transform.
__device__ __forceinline__ uint32_t morton_key(uint32_t x, uint32_t y, uint32_t z) {
    return (spread3(x) << 2) | (spread3(y) << 1) | spread3(z);
}

template <int CURVE>   // 0 Hilbert, 1 Morton
__global__ __launch_bounds__(KEYS_THREADS) void keys_kernel(const float* __restrict__ pos, int n, float3 scale,
                                                            float3 L, int bits, int npass,
                                                            unsigned long long* __restrict__ elems,
                                                            unsigned* __restrict__ hist, int32_t* status,
                                                            const int32_t* gate, int want) {
    // gate: when given, the kernel runs only if *gate == want
    pdl_wait();
    if (gate && *gate != want) return;
    __shared__ unsigned sh[MAX_PASSES][RADIX];
    __shared__ HilbertSmem s_ht;
    for (int k = threadIdx.x; k < MAX_PASSES * RADIX; k += blockDim.x) (&sh[0][0])[k] = 0u;
    if (CURVE == 0) load_hilbert_tables(s_ht);
    __syncthreads();
    const uint32_t top = (1u << bits) - 1u;
    bool bad = false;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float x = pos[3 * (size_t)i], y = pos[3 * (size_t)i + 1], z = pos[3 * (size_t)i + 2];
        bad |= !(x >= 0.0f && x < L.x && y >= 0.0f && y < L.y && z >= 0.0f && z < L.z);
        const uint32_t qx = quantize(x, scale.x, top), qy = quantize(y, scale.y, top), qz = quantize(z, scale.z, top);
        const uint32_t mk = morton_key(qx, qy, qz);
        const uint32_t key = CURVE == 0 ? hilbert_key_fsm(mk, bits, s_ht) : mk;
        elems[i] = ((unsigned long long)key << 32) | (unsigned)i;
        for (int p = 0; p < npass; ++p) atomicAdd(&sh[p][(key >> (8 * p)) & 0xffu], 1u);
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0 && status) atomicOr(status, TESS_DEV_BAD_INPUT);
    __syncthreads();
    for (int k = threadIdx.x; k < npass * RADIX; k += blockDim.x) {
        unsigned v = (&sh[0][0])[k];
        if (v) atomicAdd(&hist[k], v);
    }
}

// ---------------------------------------------------------------- onesweep

constexpr int SORT_THREADS = 256;
constexpr int SORT_WARPS = SORT_THREADS / 32;
#ifndef TESS_SORT_ITEMS
#define TESS_SORT_ITEMS 8
#endif
#ifndef TESS_SORT_MINB
#define TESS_SORT_MINB 6
#endif
constexpr int SORT_ITEMS = TESS_SORT_ITEMS;     // elements per thread in one sort tile
constexpr int SORT_TILE = SORT_THREADS * SORT_ITEMS;

// Exclusive scan of one value per thread over a 256-thread block.
__device__ __forceinline__ unsigned block_excl_scan256(unsigned v, unsigned* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        unsigned y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    unsigned wpre = 0;
#pragma unroll
    for (int w = 0; w < SORT_WARPS; ++w) wpre += (w < warp) ? s_warp[w] : 0u;
    __syncthreads();
    return wpre + x - v;
}

template <int ITEMS>
struct SortSharedT {
    unsigned long long elems[SORT_THREADS * ITEMS];
    unsigned wcnt[SORT_WARPS][RADIX];
    unsigned lbase[RADIX];
    unsigned long long gbase[RADIX];
    unsigned scan_tmp[SORT_WARPS];
    int tile;
};
using SortShared = SortSharedT<SORT_ITEMS>;

// One counting pass of the LSD sort over 64-bit elements: digit =
// (element >> shift) & 0xff.  n_dev, when given, holds the element count
// (the grid may then have more tiles than needed: tiles past the end return);
// gate, when given, runs the pass only if *gate == want.
template <bool FINAL, int ITEMS = SORT_ITEMS>
__global__ __launch_bounds__(SORT_THREADS, TESS_SORT_MINB) void onesweep_pass(const unsigned long long* __restrict__ in,
                                                              unsigned long long* __restrict__ out, int n, int shift,
                                                              const unsigned* __restrict__ hist,
                                                              unsigned long long* states, unsigned* tile_counter,
                                                              int32_t* status, int32_t* __restrict__ perm,
                                                              uint32_t* __restrict__ keys_out,
                                                              float4* __restrict__ pos_sorted,
                                                              const float* __restrict__ pos3, const int* n_dev,
                                                              const int32_t* gate, int want) {
    pdl_wait();
    constexpr int TILE = SORT_THREADS * ITEMS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SortSharedT<ITEMS>& S = *reinterpret_cast<SortSharedT<ITEMS>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (gate && *gate != want) return;
    if (n_dev) n = *n_dev;

    // persistent: each block takes tiles in order from the counter until none
    // is left (a block only takes a tile while it runs, so the look-back
    // never waits on a tile that has not started)
    for (;;) {
    if (tid == 0) S.tile = (int)atomicAdd(tile_counter, 1u);
    for (int k = tid; k < SORT_WARPS * RADIX; k += SORT_THREADS) (&S.wcnt[0][0])[k] = 0u;
    __syncthreads();
    const int tile = S.tile;
    const long long base = (long long)tile * TILE;
    if (base >= n) return;     // every tile is taken
    const long long wbase = base + (long long)warp * ITEMS * 32;

    unsigned long long e[ITEMS];
    unsigned rank[ITEMS];
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        const long long idx = wbase + k * 32 + lane;
        e[k] = idx < n ? in[idx] : ~0ull;
    }
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        const bool valid = (wbase + k * 32 + lane) < n;
        const unsigned d = (unsigned)(e[k] >> shift) & 0xffu;
        const unsigned act = __ballot_sync(FULL, valid);
        rank[k] = 0;
        if (valid) {
            const unsigned peers = __match_any_sync(act, d);
            const int leader = __ffs(peers) - 1;
            unsigned before = 0;
            if (lane == leader) {
                before = S.wcnt[warp][d];
                S.wcnt[warp][d] = before + __popc(peers);
            }
            before = __shfl_sync(peers, before, leader);
            rank[k] = before + __popc(peers & lanemask_lt());
        }
        __syncwarp();
    }
    __syncthreads();

    // per digit (thread = digit): exclusive offsets over warps, tile total
    unsigned dsum = 0;
#pragma unroll
    for (int w = 0; w < SORT_WARPS; ++w) {
        const unsigned c = S.wcnt[w][tid];
        S.wcnt[w][tid] = dsum;
        dsum += c;
    }
    unsigned long long* st = states + (size_t)tile * RADIX + tid;
    if (tile == 0) st_relaxed(st, ST_INC | dsum);
    else st_relaxed(st, ST_AGG | dsum);

    const unsigned lexcl = block_excl_scan256(dsum, S.scan_tmp);
    S.lbase[tid] = lexcl;
    const unsigned gtot = hist[tid];
    const unsigned gexcl = block_excl_scan256(gtot, S.scan_tmp);

    // decoupled look-back over the preceding tiles for this digit
    unsigned long long excl = 0;
    if (tile > 0) {
        int p = tile - 1;
        int spins = 0;
        bool timed_out = false;
        while (p >= 0) {
            const unsigned long long v = ld_relaxed(states + (size_t)p * RADIX + tid);
            const unsigned long long flag = v & ~ST_VAL;
            if (flag == 0) {
                if (++spins > LOOKBACK_SPIN_LIMIT) { timed_out = true; break; }
                __nanosleep(32);
                continue;
            }
            excl += v & ST_VAL;
            if (flag == ST_INC) break;
            --p;
        }
        if (timed_out && status) atomicOr(status, TESS_DEV_TIMEOUT);
        st_relaxed(st, ST_INC | ((excl + dsum) & ST_VAL));
    }
    S.gbase[tid] = (unsigned long long)gexcl + excl;
    __syncthreads();

    // digit-sorted copy of the tile in shared memory
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
        if ((wbase + k * 32 + lane) < n) {
            const unsigned d = (unsigned)(e[k] >> shift) & 0xffu;
            S.elems[S.lbase[d] + S.wcnt[warp][d] + rank[k]] = e[k];
        }
    }
    __syncthreads();

    const int tile_n = (int)min((long long)TILE, (long long)n - base);
    for (int s = tid; s < tile_n; s += SORT_THREADS) {
        const unsigned long long v = S.elems[s];
        const unsigned d = (unsigned)(v >> shift) & 0xffu;
        const unsigned long long g = S.gbase[d] + (unsigned long long)(s - (int)S.lbase[d]);
        if (!check_index((long long)g, n, status)) continue;
        if (FINAL) {
            const unsigned idx = (unsigned)v;
            perm[g] = (int32_t)idx;
            if (keys_out) keys_out[g] = (uint32_t)(v >> 32);
            if (pos_sorted) {
                const float* p = pos3 + 3 * (size_t)idx;
                pos_sorted[g] = make_float4(p[0], p[1], p[2], 0.0f);
            }
        } else {
            out[g] = v;
        }
    }
    __syncthreads();           // the next tile reuses the shared memory
    }
}

// ---------------------------------------------------------------- bucket sort (default)
//
// The default path sorts in one bucketing pass plus local sorts:
//   bucket_keys_kernel    key per atom, element (key << 32 | index), and the
//                         count of its bucket (the top bits of the key)
//   exclusive_scan        bucket offsets
//   bucket_scatter_kernel every element into its bucket (any order inside)
//   bucket_local_sort     one warp per bucket ranks its elements by the full
//                         64-bit element (rank = number of smaller elements)
//                         and writes perm / keys / float4 positions at
//                         offset + rank
// Elements are unique, so the order inside a bucket is fixed by the local
// ranks whatever order the scatter left them in.  Buckets hold about 40
// atoms; a bucket larger than BK_LOCAL_MAX (clustered input, a coarse grid)
// sets a device flag, and the LSD onesweep sort above -- launched gated on
// that flag -- then writes every output instead (no host synchronisation).

constexpr int BK_THREADS = 256;
constexpr int BK_LOCAL_MAX = 256;    // largest bucket a warp sorts (8 elements per lane)
constexpr int BK_WARPS = 8;          // warps per block of the local sort
constexpr int BK_TARGET = 40;        // mean bucket size the bucket bits aim for

// Bits of the key that name the bucket: about n / BK_TARGET buckets, at most
// the key's 3 * bits bits and 2^20 buckets.
static int bucket_bits(int n, int bits) {
    int db = 0;
    while (db < 20 && ((long long)BK_TARGET << db) < (long long)n) ++db;
    return std::min(db, 3 * bits);
}

template <int CURVE>
__global__ __launch_bounds__(BK_THREADS) void bucket_keys_kernel(const float* __restrict__ pos, int n, float3 scale,
                                                                 float3 L, int bits, int bshift,
                                                                 unsigned long long* __restrict__ elems,
                                                                 int* __restrict__ bcount, int* __restrict__ rank,
                                                                 int32_t* status) {
    __shared__ HilbertSmem s_ht;
    if (CURVE == 0) load_hilbert_tables(s_ht);
    __syncthreads();
    pdl_wait();
    const uint32_t top = (1u << bits) - 1u;
    bool bad = false;
    const int stride = gridDim.x * blockDim.x;
    const int lane = threadIdx.x & 31;
    for (int base = blockIdx.x * blockDim.x; base < n; base += stride) {
        const int i = base + (int)threadIdx.x;
        const bool valid = i < n;
        uint32_t b = 0;
        if (valid) {
            const float x = pos[3 * (size_t)i], y = pos[3 * (size_t)i + 1], z = pos[3 * (size_t)i + 2];
            bad |= !(x >= 0.0f && x < L.x && y >= 0.0f && y < L.y && z >= 0.0f && z < L.z);
            const uint32_t qx = quantize(x, scale.x, top), qy = quantize(y, scale.y, top),
                           qz = quantize(z, scale.z, top);
            // the default 10 bits with the level loop unrolled at compile time
            const uint32_t mk = morton_key(qx, qy, qz);
            const uint32_t key = CURVE == 0 ? (bits == 10 ? hilbert_key_fsm(mk, 10, s_ht) : hilbert_key_fsm(mk, bits, s_ht))
                                            : mk;
            elems[i] = ((unsigned long long)key << 32) | (unsigned)i;
            b = key >> bshift;
        }
        // one atomic per run of lanes in the same bucket; each element keeps
        // its place among the bucket's elements (any order: the local sort
        // fixes it), so the scatter needs no atomics of its own
        const WarpRun g = warp_run(b, valid);
        int r0 = 0;
        if (valid && lane == g.leader) r0 = atomicAdd(&bcount[b], g.len);
        r0 = __shfl_sync(FULL, r0, valid ? g.leader : lane);
        if (valid) rank[i] = r0 + g.rank;
    }
    if (__any_sync(FULL, bad) && lane == 0 && status) atomicOr(status, TESS_DEV_BAD_INPUT);
}

__global__ __launch_bounds__(BK_THREADS) void bucket_scatter_kernel(const unsigned long long* __restrict__ in, int n,
                                                                    int bshift, const int* __restrict__ bstart,
                                                                    const int* __restrict__ rank,
                                                                    unsigned long long* __restrict__ out,
                                                                    int32_t* status) {
    pdl_wait();
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + (int)threadIdx.x; i < n; i += stride) {
        const unsigned long long e = in[i];
        const uint32_t b = (uint32_t)(e >> 32) >> bshift;
        const long long slot = (long long)bstart[b] + rank[i];
        if (check_index(slot, n, status)) out[slot] = e;
    }
}

// One bucket of m elements (in shared memory s) with K elements per lane:
// each element's rank is the number of smaller elements, and it lands in
// slot beg + rank.  With EARLY the positions of the lane's atoms are fetched
// before the ranking, so that their (random) loads overlap it; the rare
// large buckets fetch them at the end and keep fewer registers.
template <int K, bool EARLY>
__device__ __forceinline__ void bucket_rank_write(const unsigned long long* s, int m, int beg, int lane,
                                                  const float* __restrict__ pos3, int32_t* __restrict__ perm,
                                                  uint32_t* __restrict__ keys_out, float4* __restrict__ pos_sorted,
                                                  int n, int32_t* status) {
    unsigned long long e[K];
    int r[K];
    float px[K], py[K], pz[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int t = lane + 32 * k;
        e[k] = t < m ? s[t] : ~0ull;
        r[k] = 0;
        if (EARLY && pos_sorted && t < m) {
            const unsigned idx = (unsigned)e[k];
            if (check_index(idx, n, status)) {
                const float* p = pos3 + 3 * (size_t)idx;
                px[k] = p[0];
                py[k] = p[1];
                pz[k] = p[2];
            }
        }
    }
#pragma unroll 4
    for (int t = 0; t < m; ++t) {
        const unsigned long long v = s[t];
#pragma unroll
        for (int k = 0; k < K; ++k) r[k] += v < e[k] ? 1 : 0;
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int t = lane + 32 * k;
        if (t < m && check_index((long long)beg + r[k], n, status) && check_index((unsigned)e[k], n, status)) {
            const int g = beg + r[k];
            perm[g] = (int32_t)(unsigned)e[k];
            if (keys_out) keys_out[g] = (uint32_t)(e[k] >> 32);
            if (pos_sorted) {
                if (!EARLY) {
                    const float* p = pos3 + 3 * (size_t)(unsigned)e[k];
                    px[k] = p[0];
                    py[k] = p[1];
                    pz[k] = p[2];
                }
                pos_sorted[g] = make_float4(px[k], py[k], pz[k], 0.0f);
            }
        }
    }
}

__global__ __launch_bounds__(BK_WARPS * 32, 4) void bucket_local_sort(const unsigned long long* __restrict__ elems,
                                                                   const int* __restrict__ bstart, int nb,
                                                                   const float* __restrict__ pos3,
                                                                   int32_t* __restrict__ perm,
                                                                   uint32_t* __restrict__ keys_out,
                                                                   float4* __restrict__ pos_sorted,
                                                                   int32_t* fallback, int n, int32_t* status) {
    pdl_wait();
    __shared__ unsigned long long s_el[BK_WARPS][BK_LOCAL_MAX];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long* s = s_el[warp];
    for (int b = blockIdx.x * BK_WARPS + warp; b < nb; b += gridDim.x * BK_WARPS) {
        const int beg = bstart[b], m = bstart[b + 1] - beg;
        if (m == 0) continue;
        if (m > BK_LOCAL_MAX) {
            if (lane == 0) atomicOr(fallback, 1);
            continue;
        }
        for (int t = lane; t < m; t += 32) s[t] = elems[beg + t];
        __syncwarp();
        if (m <= 32) bucket_rank_write<1, true>(s, m, beg, lane, pos3, perm, keys_out, pos_sorted, n, status);
        else if (m <= 64) bucket_rank_write<2, true>(s, m, beg, lane, pos3, perm, keys_out, pos_sorted, n, status);
        else if (m <= 128) bucket_rank_write<4, false>(s, m, beg, lane, pos3, perm, keys_out, pos_sorted, n, status);
        else bucket_rank_write<8, false>(s, m, beg, lane, pos3, perm, keys_out, pos_sorted, n, status);
        __syncwarp();
    }
}

// Zeroes `words` 64-bit words when *gate == want (the fallback's state).
__global__ void zero_if_kernel(unsigned long long* p, size_t words, const int32_t* gate, int want) {
    pdl_wait();
    if (*gate != want) return;
    for (size_t k = blockIdx.x * (size_t)blockDim.x + threadIdx.x; k < words; k += (size_t)gridDim.x * blockDim.x)
        p[k] = 0ull;
}

// ---------------------------------------------------------------- host

static int passes_for(int bits) { return (3 * bits + 7) / 8; }
static long long tiles_for(int n) { return ((long long)n + SORT_TILE - 1) / SORT_TILE; }

struct SortLayout {
    unsigned long long* a;
    unsigned long long* b;
    unsigned* hist;          // [MAX_PASSES][RADIX]
    unsigned* counters;      // [MAX_PASSES]
    unsigned long long* states;  // [MAX_PASSES][tiles][RADIX]
    int32_t* status;
    size_t zero_begin, zero_bytes, total;
};

static SortLayout sort_layout(void* ws, int n) {
    Carve c(ws);
    SortLayout L{};
    L.a = c.take<unsigned long long>((size_t)n);
    L.b = c.take<unsigned long long>((size_t)n);
    // the zeroed region: histograms, tile counters, tile states, status
    c.off = align_up(c.off, 256);
    L.zero_begin = c.off;
    L.hist = c.take<unsigned>(MAX_PASSES * RADIX);
    L.counters = c.take<unsigned>(MAX_PASSES);
    L.status = c.take<int32_t>(1);
    L.states = c.take<unsigned long long>((size_t)MAX_PASSES * tiles_for(n) * RADIX);
    L.zero_bytes = c.off - L.zero_begin;
    L.total = align_up(c.off, 256);
    return L;
}

static float3 grid_scale(tess_box box, int bits) {
    const float g = (float)(1u << bits);
    return make_float3(g / box.lx, g / box.ly, g / box.lz);   // fp32 IEEE divisions
}

static int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// The full sort's launches over a zeroed layout L; with a gate, every kernel
// runs only if *gate == want.
static void sfc_sort_launch(const float* pos, int n, tess_box box, int bits, int curve, const SortLayout& L,
                            int32_t* perm, uint32_t* keys_sorted, float* pos_sorted, int32_t* status,
                            const int32_t* gate, int want, cudaStream_t s) {
    const float3 scale = grid_scale(box, bits);
    const int npass = passes_for(bits);
    const int sms = sm_count();
    {
        StageScope sc(ST_KEYS, s);
        const int blocks = (int)std::min<long long>(((long long)n + KEYS_THREADS - 1) / KEYS_THREADS, (long long)sms * 8);
        if (curve == 0)
            launch_pdl(keys_kernel<0>, dim3(blocks), dim3(KEYS_THREADS), 0, s, pos, n, scale,
                       make_float3(box.lx, box.ly, box.lz), bits, npass, L.a, L.hist, status, gate, want);
        else
            launch_pdl(keys_kernel<1>, dim3(blocks), dim3(KEYS_THREADS), 0, s, pos, n, scale,
                       make_float3(box.lx, box.ly, box.lz), bits, npass, L.a, L.hist, status, gate, want);
        count_launch();
    }
    {
        StageScope sc(ST_SORT, s);
        const long long tiles = tiles_for(n);
        // persistent passes: at most the resident blocks, each looping over tiles
        const unsigned grid = (unsigned)std::min<long long>(tiles, (long long)sms * TESS_SORT_MINB);
        const size_t smem = sizeof(SortShared);
        static_assert(sizeof(SortShared) <= 48 * 1024, "sort tile must fit the default shared-memory limit");
        unsigned long long* src = L.a;
        unsigned long long* dst = L.b;
        for (int p = 0; p < npass; ++p) {
            unsigned long long* states = L.states + (size_t)p * tiles * RADIX;
            // each pass follows a kernel (the keys or the previous pass)
            if (p == npass - 1) {
                launch_pdl(onesweep_pass<true>, dim3(grid), dim3(SORT_THREADS), smem, s, src, nullptr, n, 32 + 8 * p,
                           L.hist + p * RADIX, states, L.counters + p, status, perm, keys_sorted,
                           reinterpret_cast<float4*>(pos_sorted), pos, nullptr, gate, want);
            } else {
                launch_pdl(onesweep_pass<false>, dim3(grid), dim3(SORT_THREADS), smem, s, src, dst, n, 32 + 8 * p,
                           L.hist + p * RADIX, states, L.counters + p, status, nullptr, nullptr, nullptr, nullptr,
                           nullptr, gate, want);
            }
            count_launch();
            std::swap(src, dst);
        }
    }
}

// Workspace of the default sort: the LSD sort's layout (its two element
// buffers also carry the bucket pass), then the bucket counts / offsets.
struct BucketLayout {
    SortLayout lsd;
    int* bcount;             // [nb] counts
    int* rank;               // [n] place of each element in its bucket (in the LSD sort's
                             // look-back states, which the fallback zeroes before use)
    int32_t* flag;           // 1: some bucket too large for the local sort
    unsigned long long* scan_state;   // look-back words of the offset scan
    int* bstart;             // [nb + 1]
    size_t zero_begin, zero_bytes, total;
};

static BucketLayout bucket_layout(void* ws, int n) {
    BucketLayout B{};
    B.lsd = sort_layout(ws, n);
    Carve c(ws);
    c.off = B.lsd.total;
    const long long nb = 1LL << bucket_bits(n, 10);
    c.off = align_up(c.off, 256);
    B.zero_begin = c.off;
    B.bcount = c.take<int>((size_t)nb);
    B.flag = c.take<int32_t>(1);
    B.scan_state = c.take<unsigned long long>((size_t)scan_state_len(nb));
    B.zero_bytes = c.off - B.zero_begin;
    B.bstart = c.take<int>((size_t)nb + 1);
    B.total = align_up(c.off, 256);
    // 4 passes x tiles of 2048 x 256 eight-byte states hold n ints
    static_assert((size_t)MAX_PASSES * RADIX * 8 >= (size_t)SORT_TILE * 4, "rank storage");
    B.rank = reinterpret_cast<int*>(B.lsd.states);
    return B;
}

size_t hilbert_sort_workspace(int n) {
    if (n <= 0) return 0;
    return bucket_layout(nullptr, n).total;
}

tess_status sfc_sort(const float* pos, int n, tess_box box, int bits, int curve, void* ws, size_t ws_bytes,
                     int32_t* perm, uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s) {
    if (n <= 0 || !pos || !perm || !ws || bits < 1 || bits > 10) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (pos_sorted && !aligned(pos_sorted, 16)) return TESS_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return TESS_ERR_INVALID_ARG;
    BucketLayout B = bucket_layout(ws, n);
    if (ws_bytes < B.total) return TESS_ERR_WORKSPACE_TOO_SMALL;
    const SortLayout& L = B.lsd;
    int32_t* status = dev_status ? dev_status : L.status;

    const int db = bucket_bits(n, bits);
    const long long nb = 1LL << db;
    const int bshift = 3 * bits - db;
    const float3 scale = grid_scale(box, bits);
    const float3 Lb = make_float3(box.lx, box.ly, box.lz);
    const int sms = sm_count();
    const int blocks = (int)std::min<long long>(((long long)n + BK_THREADS - 1) / BK_THREADS, (long long)sms * 8);

    zero2(reinterpret_cast<unsigned*>(static_cast<char*>(ws) + B.zero_begin), B.zero_bytes / 4,
          reinterpret_cast<unsigned*>(dev_status), dev_status ? 1 : 0, sms, s);
    {
        StageScope sc(ST_KEYS, s);
        if (curve == 0)
            launch_pdl(bucket_keys_kernel<0>, dim3(blocks), dim3(BK_THREADS), 0, s, pos, n, scale, Lb, bits, bshift,
                       L.a, B.bcount, B.rank, status);
        else
            launch_pdl(bucket_keys_kernel<1>, dim3(blocks), dim3(BK_THREADS), 0, s, pos, n, scale, Lb, bits, bshift,
                       L.a, B.bcount, B.rank, status);
        count_launch();
    }
    {
        StageScope sc(ST_SORT, s);
        exclusive_scan(B.bcount, nb, B.scan_state, B.bstart, status, sms, s);
        launch_pdl(bucket_scatter_kernel, dim3(blocks), dim3(BK_THREADS), 0, s, (const unsigned long long*)L.a, n,
                   bshift, (const int*)B.bstart, (const int*)B.rank, L.b, status);
        const int lblocks = (int)std::min<long long>((nb + BK_WARPS - 1) / BK_WARPS, (long long)sms * 16);
        launch_pdl(bucket_local_sort, dim3(lblocks), dim3(BK_WARPS * 32), 0, s, (const unsigned long long*)L.b,
                   (const int*)B.bstart, (int)nb, pos, perm, keys_sorted, reinterpret_cast<float4*>(pos_sorted),
                   B.flag, n, status);
        count_launch(2);
        // a bucket too large for the local sort: the LSD sort, gated on the flag
        launch_pdl(zero_if_kernel, dim3(sms * 2), dim3(256), 0, s,
                   reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.zero_begin),
                   (size_t)(L.zero_bytes / 8), (const int32_t*)B.flag, 1);
        count_launch();
    }
    sfc_sort_launch(pos, n, box, bits, curve, L, perm, keys_sorted, pos_sorted, status, B.flag, 1, s);
    return launch_status();
}

tess_status hilbert_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                         uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s) {
    return sfc_sort(pos, n, box, bits, 0, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status, s);
}

tess_status morton_sort(const float* pos, int n, tess_box box, int bits, void* ws, size_t ws_bytes, int32_t* perm,
                        uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s) {
    return sfc_sort(pos, n, box, bits, 1, ws, ws_bytes, perm, keys_sorted, pos_sorted, dev_status, s);
}

// ---------------------------------------------------------------- incremental resort
//
// Re-sorts atoms that have moved since an earlier sort, starting from that
// sort's order (perm_prev, keys_prev).  Each atom's composite element
// (key << 32 | index) is unique, so the sorted order is unique and any exact
// method reproduces the full sort.  Between rebuilds most atoms move by a
// fraction of a grid cell, so their new key stays inside the range of old
// keys of their old neighbors in the order: such "local" atoms (S) can only
// be out of order with atoms at most 2 * RS_W old ranks away and are sorted
// by two phases of block sorts of RS_BLK elements (the second offset by half
// a block).  The others (O, atoms whose key jumped along the curve: the
// curve's neighboring cells can be far apart in key) are few; they are radix
// sorted by the full 64-bit element and merged in by binary search.  Every
// assumption is checked on the device: perm_prev must be a permutation, O
// must fit its buffer and S must come out strictly increasing; otherwise a
// device flag switches to the full sort, whose kernels are launched gated on
// that flag (no host synchronisation either way).

constexpr int RS_W = 64;                 // old-rank window of the key range
constexpr int RS_D = 2 * RS_W;           // displacement bound of local atoms
constexpr int RS_BLK = 2 * RS_D;         // 256 elements per block sort (one warp, 8 per lane)
constexpr int RS_THREADS = 256;
constexpr int RS_TILE = 1024;            // elements per classify / compact block

struct ResortCtl {
    int32_t fallback;    // 1: the fast path's assumptions failed, run the full sort
    int32_t m_local;     // |S|
    int32_t m_out;       // |O|
    int32_t pad;
};

__device__ __forceinline__ int block_sum256(int v, int* s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < RS_THREADS / 32; ++w) t += s_red[w];
    __syncthreads();
    return t;
}

// Composite elements in the previous order, local flags, per-tile local
// counts.  An index of perm_prev outside [0, n) switches to the full sort;
// a repeated index is caught later (two equal elements meet in the runs'
// order checks or in the merge), so perm_prev is a permutation whenever
// the fast path completes.
__global__ __launch_bounds__(RS_THREADS) void resort_classify(const float* __restrict__ pos, int n, float3 scale,
                                                              float3 L, int bits,
                                                              const int32_t* __restrict__ perm_prev,
                                                              const uint32_t* __restrict__ keys_prev,
                                                              unsigned long long* __restrict__ elems,
                                                              uint8_t* __restrict__ local,
                                                              int* __restrict__ tile_cnt, ResortCtl* ctl,
                                                              int32_t* status) {
    __shared__ int s_red[RS_THREADS / 32];
    __shared__ HilbertSmem s_ht;
    load_hilbert_tables(s_ht);
    __syncthreads();
    const long long base = (long long)blockIdx.x * RS_TILE;
    const uint32_t top = (1u << bits) - 1u;
    constexpr int U = RS_TILE / RS_THREADS;
    int cnt = 0;
    bool bad = false, broken = false;
    int idx[U];
    float px[U], py[U], pz[U];
    uint32_t lo[U], hi[U];
    // all loads of the thread's elements first, so that their latencies overlap
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const long long k = base + u * RS_THREADS + threadIdx.x;
        idx[u] = k < n ? perm_prev[k] : 0;
        if (idx[u] < 0 || idx[u] >= n) {
            broken = true;
            idx[u] = 0;
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const long long k = base + u * RS_THREADS + threadIdx.x;
        const long long kk = k < n ? k : n - 1;
        px[u] = pos[3 * (size_t)idx[u]];
        py[u] = pos[3 * (size_t)idx[u] + 1];
        pz[u] = pos[3 * (size_t)idx[u] + 2];
        lo[u] = keys_prev[kk >= RS_W ? kk - RS_W : 0];
        hi[u] = keys_prev[kk + RS_W < n ? kk + RS_W : n - 1];
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const long long k = base + u * RS_THREADS + threadIdx.x;
        if (k >= n) break;
        const float x = px[u], y = py[u], z = pz[u];
        bad |= !(x >= 0.0f && x < L.x && y >= 0.0f && y < L.y && z >= 0.0f && z < L.z);
        const uint32_t key = hilbert_key_fsm(
            morton_key(quantize(x, scale.x, top), quantize(y, scale.y, top), quantize(z, scale.z, top)), bits, s_ht);
        elems[k] = ((unsigned long long)key << 32) | (unsigned)idx[u];
        const bool loc = key >= lo[u] && key <= hi[u];
        local[k] = loc ? 1 : 0;
        cnt += loc ? 1 : 0;
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0 && status) atomicOr(status, TESS_DEV_BAD_INPUT);
    if (broken) atomicExch(&ctl->fallback, 1);
    const int total = block_sum256(cnt, s_red);
    if (threadIdx.x == 0) tile_cnt[blockIdx.x] = total;
}

// Exclusive scan of the per-tile local counts (one block of 1024 threads);
// sizes of S and O; O larger than its buffer switches to the full sort.
__global__ __launch_bounds__(1024) void resort_scan(int* tile_cnt, int ntiles, int n, int cap_out, ResortCtl* ctl) {
    __shared__ int s_warp[32];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int per = (ntiles + 1023) / 1024;
    const int b0 = min(t * per, ntiles), b1 = min(b0 + per, ntiles);
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += tile_cnt[b];
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += s_warp[w];
    int run = wpre + x - sum;
    for (int b = b0; b < b1; ++b) {
        const int c = tile_cnt[b];
        tile_cnt[b] = run;
        run += c;
    }
    if (t == 1023) {
        const int m_local = wpre + x;
        ctl->m_local = m_local;
        ctl->m_out = n - m_local;
        if (n - m_local > cap_out) atomicExch(&ctl->fallback, 1);
    }
}

// O is radix sorted by its key bytes (stable, in O's own order); equal keys
// whose indices come out descending are caught in the merge.
// Splits the elements into S and O in order (per-tile offsets from
// resort_scan) and builds O's digit histograms.
__global__ __launch_bounds__(RS_THREADS) void resort_compact(const unsigned long long* __restrict__ elems,
                                                             const uint8_t* __restrict__ local, int n,
                                                             const int* __restrict__ tile_off,
                                                             unsigned long long* __restrict__ S,
                                                             unsigned long long* __restrict__ O, int npass,
                                                             unsigned* ohist, const ResortCtl* ctl) {
    __shared__ int s_warp[RS_THREADS / 32];
    __shared__ unsigned sh[2 * MAX_PASSES][RADIX];
    if (ctl->fallback) return;
    for (int k = threadIdx.x; k < 2 * MAX_PASSES * RADIX; k += RS_THREADS) (&sh[0][0])[k] = 0u;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long base = (long long)blockIdx.x * RS_TILE;
    constexpr int PER = RS_TILE / RS_THREADS;     // consecutive elements per thread
    const long long k0 = base + (long long)t * PER;
    int f[PER];
    int c = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        f[u] = (k0 + u < n) ? local[k0 + u] : 0;
        c += f[u];
    }
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int wpre = 0;
#pragma unroll
    for (int w = 0; w < RS_THREADS / 32; ++w) wpre += (w < warp) ? s_warp[w] : 0;
    const int pre_local = wpre + x - c;                          // local atoms of this tile before thread t
    const long long valid_before = min((long long)t * PER, max(0ll, (long long)n - base));
    long long si = (long long)tile_off[blockIdx.x] + pre_local;
    long long oi = (base - tile_off[blockIdx.x]) + (valid_before - pre_local);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        if (k0 + u >= n) break;
        const unsigned long long v = elems[k0 + u];
        if (f[u]) {
            S[si++] = v;
        } else {
            O[oi++] = v;
            for (int p = 0; p < npass; ++p) atomicAdd(&sh[p][(unsigned)(v >> (32 + 8 * p)) & 0xffu], 1u);
        }
    }
    __syncthreads();
    for (int k = threadIdx.x; k < npass * RADIX; k += RS_THREADS) {
        const unsigned v = (&sh[0][0])[k];
        if (v) atomicAdd(&ohist[k], v);
    }
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
    const unsigned lo = __shfl_xor_sync(FULL, (unsigned)v, m);
    const unsigned hi = __shfl_xor_sync(FULL, (unsigned)(v >> 32), m);
    return ((unsigned long long)hi << 32) | lo;
}

// Sorts blocks of S in place, one warp per block of RS_BLK elements held in
// registers (lane l holds positions 8l .. 8l+7), with a bitonic network.
// Phase 0: blocks at multiples of RS_BLK; phase 1: the same shifted by RS_D
// (the first block is [0, RS_D)).  Missing elements are padded with the
// largest value, so they sort last and are not written back.  Global memory
// is read and written in coalesced stripes (lane l: positions l + 32r) and
// transposed through shared memory, skewed by one slot per 8 against bank
// conflicts.
__device__ __forceinline__ int rs_skew(int p) { return p + (p >> 3); }

template <int PHASE>
__global__ __launch_bounds__(RS_THREADS) void resort_block_sort(unsigned long long* __restrict__ S,
                                                                const ResortCtl* ctl) {
    __shared__ unsigned long long sx[RS_THREADS / 32][RS_BLK + RS_BLK / 8];
    if (ctl->fallback) return;
    const int m = ctl->m_local;
    const int lane = threadIdx.x & 31;
    unsigned long long* t = sx[threadIdx.x >> 5];
    const long long wg = (long long)blockIdx.x * (RS_THREADS / 32) + (threadIdx.x >> 5);
    // phase 1: block w >= 1 starts at RS_D + (w - 1) * RS_BLK; its halves are
    // the sorted second half of one phase-0 block and the sorted first half
    // of the next (the first RS_D elements are a sorted half already)
    if (PHASE == 1 && wg == 0) return;
    const long long start = PHASE == 0 ? wg * RS_BLK : RS_D + (wg - 1) * RS_BLK;
    if (start >= m) return;
    const long long len = min((long long)RS_BLK, (long long)m - start);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int p = 32 * r + lane;
        t[rs_skew(p)] = p < len ? S[start + p] : ~0ull;
    }
    __syncwarp();
    unsigned long long x[8];
    if (PHASE == 0) {
#pragma unroll
        for (int r = 0; r < 8; ++r) x[r] = t[rs_skew(8 * lane + r)];
    } else {
        // second half reversed: the block becomes one bitonic sequence
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int p = 8 * lane + r;
            x[r] = t[rs_skew(p < RS_D ? p : 3 * RS_D - 1 - p)];
        }
    }
#pragma unroll
    for (int k = PHASE == 0 ? 2 : RS_BLK; k <= RS_BLK; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 8) {
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int p = 8 * lane + r;
                    const unsigned long long y = shfl_xor_u64(x[r], j >> 3);
                    const bool lower = (p & j) == 0, asc = (p & k) == 0;
                    x[r] = (lower == asc) ? (x[r] < y ? x[r] : y) : (x[r] < y ? y : x[r]);
                }
            } else {
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int q = r ^ j;
                    if (q > r) {
                        const bool asc = ((8 * lane + r) & k) == 0;
                        const unsigned long long a = x[r], b = x[q];
                        const bool sw = asc ? (a > b) : (a < b);
                        x[r] = sw ? b : a;
                        x[q] = sw ? a : b;
                    }
                }
            }
        }
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 8; ++r) t[rs_skew(8 * lane + r)] = x[r];
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int p = 32 * r + lane;
        if (p < len) S[start + p] = t[rs_skew(p)];
    }
}

// S must be strictly increasing after the block sorts; otherwise fall back.
__global__ __launch_bounds__(RS_THREADS) void resort_check(const unsigned long long* __restrict__ S, ResortCtl* ctl) {
    if (ctl->fallback) return;
    const long long m = ctl->m_local;
    bool bad = false;
    for (long long k = (long long)blockIdx.x * RS_THREADS + threadIdx.x; k + 1 < m; k += (long long)gridDim.x * RS_THREADS)
        bad |= !(S[k] < S[k + 1]);
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0) atomicExch(&ctl->fallback, 1);
}

// Number of elements of a[0..m) below v (a strictly increasing).
__device__ __forceinline__ long long count_below(const unsigned long long* __restrict__ a, long long m,
                                                 unsigned long long v) {
    long long lo = 0, hi = m;
    while (lo < hi) {
        const long long mid = (lo + hi) >> 1;
        if (a[mid] < v) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// Number of entries of c[0..m) that are <= t (c non-decreasing).
template <class T>
__device__ __forceinline__ int count_le(const T* c, int m, long long t) {
    int lo = 0, hi = m;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((long long)c[mid] <= t) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void write_sorted(long long g, unsigned long long v, const float* __restrict__ pos3,
                                             int32_t* __restrict__ perm, uint32_t* __restrict__ keys_out,
                                             float4* __restrict__ pos_sorted) {
    const unsigned idx = (unsigned)v;
    perm[g] = (int32_t)idx;
    if (keys_out) keys_out[g] = (uint32_t)(v >> 32);
    if (pos_sorted) {
        const float* p = pos3 + 3 * (size_t)idx;
        pos_sorted[g] = make_float4(p[0], p[1], p[2], 0.0f);
    }
}

// Merge, part 1: each element of O (rank r) counts the elements of S below
// it, c[r], and lands in slot r + c[r].  c is non-decreasing in r.  O must
// be strictly increasing (equal keys in index order, no repeated element)
// and share no element with S; otherwise the full sort runs (it rewrites
// every output slot, and every slot written here is below n).
__global__ __launch_bounds__(RS_THREADS) void resort_merge_out(const unsigned long long* __restrict__ S,
                                                               const unsigned long long* __restrict__ Os,
                                                               int* __restrict__ c_out, const ResortCtl* ctl,
                                                               const float* __restrict__ pos3,
                                                               int32_t* __restrict__ perm,
                                                               uint32_t* __restrict__ keys_out,
                                                               float4* __restrict__ pos_sorted, ResortCtl* ctl_w) {
    if (ctl->fallback) return;
    const long long ms = ctl->m_local, mo = ctl->m_out;
    bool bad = false;
    for (long long r = (long long)blockIdx.x * RS_THREADS + threadIdx.x; r < mo; r += (long long)gridDim.x * RS_THREADS) {
        const unsigned long long v = Os[r];
        const long long c = count_below(S, ms, v);
        bad |= (c < ms && S[c] == v) || (r + 1 < mo && !(v < Os[r + 1]));
        c_out[r] = (int)c;
        if (check_index(r + c, ms + mo, nullptr)) write_sorted(r + c, v, pos3, perm, keys_out, pos_sorted);
        else bad = true;          // checked builds: the full sort rewrites every slot
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0) atomicExch(&ctl_w->fallback, 1);
}

constexpr int RS_MERGE_SPAN = 4096;      // S elements per block in merge part 2
constexpr int RS_MERGE_STAGE = 1024;     // O counts staged in shared memory per block

// Merge, part 2: element t of S lands in slot t + #{r : c[r] <= t}.  A block
// owns S[t0, t0 + RS_MERGE_SPAN); the c[r] that fall in that span are
// staged in shared memory (searched in global memory if there are more).
__global__ __launch_bounds__(RS_THREADS) void resort_merge_local(const unsigned long long* __restrict__ S,
                                                                 const int* __restrict__ c_out, const ResortCtl* ctl,
                                                                 const float* __restrict__ pos3,
                                                                 int32_t* __restrict__ perm,
                                                                 uint32_t* __restrict__ keys_out,
                                                                 float4* __restrict__ pos_sorted, int32_t* status) {
    __shared__ int s_c[RS_MERGE_STAGE];
    __shared__ int s_lo, s_hi;
    if (ctl->fallback) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && status) atomicOr(status, TESS_DEV_FULL_SORT);
        return;
    }
    const long long ms = ctl->m_local;
    const int mo = ctl->m_out;
    for (long long t0 = (long long)blockIdx.x * RS_MERGE_SPAN; t0 < ms; t0 += (long long)gridDim.x * RS_MERGE_SPAN) {
        const long long t1 = min(ms, t0 + RS_MERGE_SPAN);
        if (threadIdx.x == 0) {
            s_lo = count_le(c_out, mo, t0 - 1);        // O elements below S[t0]
            s_hi = count_le(c_out, mo, t1 - 1);
        }
        __syncthreads();
        const int lo = s_lo, cnt = s_hi - s_lo;
        const bool staged = cnt <= RS_MERGE_STAGE;
        if (staged)
            for (int k = threadIdx.x; k < cnt; k += RS_THREADS) s_c[k] = c_out[lo + k];
        __syncthreads();
        constexpr int U = 4;
        for (long long tb = t0 + threadIdx.x; tb < t1; tb += U * RS_THREADS) {
            unsigned long long v[U];
            float3 q[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long t = tb + u * RS_THREADS;
                v[u] = t < t1 ? S[t] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float* p = pos3 + 3 * (size_t)(unsigned)v[u];
                q[u] = make_float3(p[0], p[1], p[2]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long t = tb + u * RS_THREADS;
                if (t >= t1) break;
                const int below = staged ? lo + count_le(s_c, cnt, t) : count_le(c_out, mo, t);
                const long long g = t + below;
                if (!check_index(g, ctl->m_local + ctl->m_out, status)) continue;
                perm[g] = (int32_t)(unsigned)v[u];
                if (keys_out) keys_out[g] = (uint32_t)(v[u] >> 32);
                if (pos_sorted) pos_sorted[g] = make_float4(q[u].x, q[u].y, q[u].z, 0.0f);
            }
        }
        __syncthreads();
    }
}

struct ResortLayout {
    SortLayout full;            // the full sort's buffers (fallback); full.a / full.b also hold elems / S
    unsigned long long* o0;
    unsigned long long* o1;
    int* c_out;                 // [cap_out] S elements below each O element
    uint8_t* local;
    int* tile_cnt;
    unsigned* ohist;            // [2 * MAX_PASSES][RADIX]
    unsigned* ocounters;        // [2 * MAX_PASSES]
    unsigned long long* ostates;  // [2 * MAX_PASSES][out tiles][RADIX]
    ResortCtl* ctl;
    size_t zero_begin, zero_bytes, total;
    int cap_out;
};

static int resort_cap_out(int n) { return n / 8 + 1024; }

static ResortLayout resort_layout(void* ws, int n) {
    ResortLayout R{};
    R.full = sort_layout(ws, n);
    Carve c(ws);
    c.off = R.full.total;
    R.cap_out = resort_cap_out(n);
    R.o0 = c.take<unsigned long long>((size_t)R.cap_out);
    R.o1 = c.take<unsigned long long>((size_t)R.cap_out);
    R.c_out = c.take<int>((size_t)R.cap_out);
    R.local = c.take<uint8_t>((size_t)n);
    const long long ntiles = ((long long)n + RS_TILE - 1) / RS_TILE;
    R.tile_cnt = c.take<int>((size_t)ntiles);
    c.off = align_up(c.off, 256);
    R.zero_begin = c.off;
    R.ohist = c.take<unsigned>(2 * MAX_PASSES * RADIX);
    R.ocounters = c.take<unsigned>(2 * MAX_PASSES);
    R.ctl = c.take<ResortCtl>(1);
    R.ostates = c.take<unsigned long long>((size_t)2 * MAX_PASSES * (((size_t)R.cap_out + 1023) / 1024) * RADIX);
    R.zero_bytes = c.off - R.zero_begin;
    R.total = align_up(c.off, 256);
    return R;
}

size_t hilbert_resort_workspace(int n) {
    if (n <= 0) return 0;
    return resort_layout(nullptr, n).total;
}

tess_status hilbert_resort(const float* pos, int n, tess_box box, int bits, const int32_t* perm_prev,
                           const uint32_t* keys_prev, void* ws, size_t ws_bytes, int32_t* perm,
                           uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s) {
    if (n <= 0 || !pos || !perm || !perm_prev || !keys_prev || !ws || bits < 1 || bits > 10)
        return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (pos_sorted && !aligned(pos_sorted, 16)) return TESS_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return TESS_ERR_INVALID_ARG;
    ResortLayout R = resort_layout(ws, n);
    if (ws_bytes < R.total) return TESS_ERR_WORKSPACE_TOO_SMALL;
    int32_t* status = dev_status ? dev_status : R.full.status;
    char* w = static_cast<char*>(ws);
    cudaMemsetAsync(w + R.full.zero_begin, 0, R.full.zero_bytes, s);
    cudaMemsetAsync(w + R.zero_begin, 0, R.zero_bytes, s);
    if (dev_status) cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s);

    const int sms = sm_count();
    const int ntiles = (int)(((long long)n + RS_TILE - 1) / RS_TILE);
    const int npass = passes_for(bits);
    unsigned long long* elems = R.full.a;
    unsigned long long* S = R.full.b;
    {
        StageScope sc(ST_RESORT, s);
        resort_classify<<<ntiles, RS_THREADS, 0, s>>>(pos, n, grid_scale(box, bits),
                                                      make_float3(box.lx, box.ly, box.lz), bits, perm_prev,
                                                      keys_prev, elems, R.local, R.tile_cnt, R.ctl, status);
        resort_scan<<<1, 1024, 0, s>>>(R.tile_cnt, ntiles, n, R.cap_out, R.ctl);
        resort_compact<<<ntiles, RS_THREADS, 0, s>>>(elems, R.local, n, R.tile_cnt, S, R.o0, npass, R.ohist, R.ctl);
        const long long warps1 = ((long long)n + RS_BLK - 1) / RS_BLK + 1;
        const int bs_blocks = (int)((warps1 + RS_THREADS / 32 - 1) / (RS_THREADS / 32));
        resort_block_sort<0><<<bs_blocks, RS_THREADS, 0, s>>>(S, R.ctl);
        resort_block_sort<1><<<bs_blocks, RS_THREADS, 0, s>>>(S, R.ctl);
        resort_check<<<sms * 4, RS_THREADS, 0, s>>>(S, R.ctl);
        count_launch(6);
        // O: LSD radix sort by key, gated on the fast path
        constexpr int O_ITEMS = 4;     // small tiles: O is short, so more tiles run side by side
        const long long otiles = ((long long)R.cap_out + SORT_THREADS * O_ITEMS - 1) / (SORT_THREADS * O_ITEMS);
        unsigned long long* src = R.o0;
        unsigned long long* dst = R.o1;
        for (int p = 0; p < npass; ++p) {
            onesweep_pass<false, O_ITEMS><<<(unsigned)otiles, SORT_THREADS, sizeof(SortSharedT<O_ITEMS>), s>>>(
                src, dst, R.cap_out, 32 + 8 * p, R.ohist + p * RADIX,
                R.ostates + (size_t)p * otiles * RADIX, R.ocounters + p, status, nullptr, nullptr, nullptr, nullptr,
                &R.ctl->m_out, &R.ctl->fallback, 0);
            std::swap(src, dst);
        }
        count_launch(npass);
        resort_merge_out<<<sms * 2, RS_THREADS, 0, s>>>(S, src, R.c_out, R.ctl, pos, perm, keys_sorted,
                                                        reinterpret_cast<float4*>(pos_sorted), R.ctl);
        resort_merge_local<<<sms * 8, RS_THREADS, 0, s>>>(S, R.c_out, R.ctl, pos, perm, keys_sorted,
                                                          reinterpret_cast<float4*>(pos_sorted), status);
        count_launch(2);
    }
    // the full sort, run only when the fast path's checks failed
    sfc_sort_launch(pos, n, box, bits, 0, R.full, perm, keys_sorted, pos_sorted, status, &R.ctl->fallback, 1, s);
    return launch_status();
}

// ---------------------------------------------------------------- look-back timeout probe
//
// Exercises the bounded wait of the counting pass: one block runs tile 1 of
// a two-tile pass (the tile counter starts at 1) while tile 0 never runs, so
// the look-back finds tile 0 unpublished, gives up after LOOKBACK_SPIN_LIMIT
// polls and sets TESS_DEV_TIMEOUT; the pass then completes.  All keys are 0
// and the digit histogram counts both tiles, so every write stays inside
// the workspace.  For tests of the timeout path; its output means nothing.

struct ProbeLayout {
    unsigned long long* in;
    unsigned long long* out;
    unsigned* hist;
    unsigned long long* states;
    unsigned* counter;
    size_t total;
};

static ProbeLayout probe_layout(void* ws) {
    Carve c(ws);
    ProbeLayout P{};
    P.in = c.take<unsigned long long>(2 * SORT_TILE);
    P.out = c.take<unsigned long long>(2 * SORT_TILE);
    P.hist = c.take<unsigned>(RADIX);
    P.states = c.take<unsigned long long>(2 * RADIX);
    P.counter = c.take<unsigned>(1);
    P.total = align_up(c.off, 256);
    return P;
}

__global__ void probe_init(unsigned* hist, unsigned* counter, unsigned n) {
    hist[0] = n;          // every key is 0: digit 0 holds all elements
    *counter = 1;         // the only block takes tile 1
}

size_t lookback_probe_workspace() { return probe_layout(nullptr).total; }

tess_status lookback_timeout_probe(void* ws, size_t ws_bytes, int32_t* status, cudaStream_t s) {
    if (!ws || !status || !aligned(ws, 256)) return TESS_ERR_INVALID_ARG;
    ProbeLayout P = probe_layout(ws);
    if (ws_bytes < P.total) return TESS_ERR_WORKSPACE_TOO_SMALL;
    cudaMemsetAsync(ws, 0, P.total, s);
    cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    probe_init<<<1, 1, 0, s>>>(P.hist, P.counter, 2u * SORT_TILE);
    onesweep_pass<false><<<1, SORT_THREADS, sizeof(SortShared), s>>>(
        P.in, P.out, 2 * SORT_TILE, 32, P.hist, P.states, P.counter, status, nullptr, nullptr, nullptr, nullptr,
        nullptr, nullptr, 0);
    count_launch(2);
    return launch_status();
}

}  // namespace tess
