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
#include "common.cuh"

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

// 3-D Hilbert index of grid point (x, y, z) with `bits` bits per axis,
// following Skilling's transform ("Programming the Hilbert curve", 2004):
// undo the sub-cube rotations/reflections level by level from the top, Gray
// encode across axes, fold in the parity of the last axis, and interleave
// the three words most-significant level first (x's bit highest in each
// triple).  Written branch-free: each per-level choice between "invert" and
// "exchange" becomes a mask, and the parity fold is a suffix-XOR scan.
__device__ __forceinline__ uint32_t hilbert_key(uint32_t x, uint32_t y, uint32_t z, int bits) {
    for (int l = bits - 1; l >= 1; --l) {
        const uint32_t low = (1u << l) - 1u;
        x ^= low & (0u - ((x >> l) & 1u));              // axis 0: invert or no-op
        uint32_t m = 0u - ((y >> l) & 1u);
        uint32_t t = (x ^ y) & low & ~m;                // exchange part (bit clear)
        x ^= (low & m) ^ t;                             // invert (bit set) or exchange
        y ^= t;
        m = 0u - ((z >> l) & 1u);
        t = (x ^ z) & low & ~m;
        x ^= (low & m) ^ t;
        z ^= t;
    }
    y ^= x;
    z ^= y;
    // bit k of the fold = XOR of z's bits above k
    uint32_t f = z >> 1;
    f ^= f >> 1;
    f ^= f >> 2;
    f ^= f >> 4;
    f ^= f >> 8;
    x ^= f;
    y ^= f;
    z ^= f;
    return (spread3(x) << 2) | (spread3(y) << 1) | spread3(z);
}

// Grid cell of one coordinate: floor(x * scale) with one fp32 multiply,
// clamped into [0, top]; products below 1 (negative, NaN) give 0.
__device__ __forceinline__ uint32_t quantize(float x, float scale, uint32_t top) {
    float prod = __fmul_rn(x, scale);
    if (!(prod >= 1.0f)) return 0u;
    float fl = floorf(prod);
    return fl >= (float)top ? top : (uint32_t)fl;
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
                                                            unsigned* __restrict__ hist, int32_t* status) {
    __shared__ unsigned sh[MAX_PASSES][RADIX];
    for (int k = threadIdx.x; k < MAX_PASSES * RADIX; k += blockDim.x) (&sh[0][0])[k] = 0u;
    __syncthreads();
    const uint32_t top = (1u << bits) - 1u;
    bool bad = false;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float x = pos[3 * (size_t)i], y = pos[3 * (size_t)i + 1], z = pos[3 * (size_t)i + 2];
        bad |= !(x >= 0.0f && x < L.x && y >= 0.0f && y < L.y && z >= 0.0f && z < L.z);
        const uint32_t qx = quantize(x, scale.x, top), qy = quantize(y, scale.y, top), qz = quantize(z, scale.z, top);
        const uint32_t key = CURVE == 0 ? hilbert_key(qx, qy, qz, bits) : morton_key(qx, qy, qz);
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
constexpr int SORT_ITEMS = 16;
constexpr int SORT_TILE = SORT_THREADS * SORT_ITEMS;
constexpr unsigned long long ST_AGG = 1ull << 62;
constexpr unsigned long long ST_INC = 2ull << 62;
constexpr unsigned long long ST_VAL = (1ull << 62) - 1ull;
constexpr int LOOKBACK_SPIN_LIMIT = 1 << 22;

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

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

struct SortShared {
    unsigned long long elems[SORT_TILE];
    unsigned wcnt[SORT_WARPS][RADIX];
    unsigned lbase[RADIX];
    unsigned long long gbase[RADIX];
    unsigned scan_tmp[SORT_WARPS];
    int tile;
};

template <bool FINAL>
__global__ __launch_bounds__(SORT_THREADS, 3) void onesweep_pass(const unsigned long long* __restrict__ in,
                                                              unsigned long long* __restrict__ out, int n, int shift,
                                                              const unsigned* __restrict__ hist,
                                                              unsigned long long* states, unsigned* tile_counter,
                                                              int32_t* status, int32_t* __restrict__ perm,
                                                              uint32_t* __restrict__ keys_out,
                                                              float4* __restrict__ pos_sorted,
                                                              const float* __restrict__ pos3) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SortShared& S = *reinterpret_cast<SortShared*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) S.tile = (int)atomicAdd(tile_counter, 1u);
    for (int k = tid; k < SORT_WARPS * RADIX; k += SORT_THREADS) (&S.wcnt[0][0])[k] = 0u;
    __syncthreads();
    const int tile = S.tile;
    const long long base = (long long)tile * SORT_TILE;
    const long long wbase = base + (long long)warp * SORT_ITEMS * 32;

    unsigned long long e[SORT_ITEMS];
    unsigned rank[SORT_ITEMS];
#pragma unroll
    for (int k = 0; k < SORT_ITEMS; ++k) {
        const long long idx = wbase + k * 32 + lane;
        e[k] = idx < n ? in[idx] : ~0ull;
    }
#pragma unroll
    for (int k = 0; k < SORT_ITEMS; ++k) {
        const bool valid = (wbase + k * 32 + lane) < n;
        const unsigned d = (unsigned)(e[k] >> (32 + shift)) & 0xffu;
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
    for (int k = 0; k < SORT_ITEMS; ++k) {
        if ((wbase + k * 32 + lane) < n) {
            const unsigned d = (unsigned)(e[k] >> (32 + shift)) & 0xffu;
            S.elems[S.lbase[d] + S.wcnt[warp][d] + rank[k]] = e[k];
        }
    }
    __syncthreads();

    const int tile_n = (int)min((long long)SORT_TILE, (long long)n - base);
    for (int s = tid; s < tile_n; s += SORT_THREADS) {
        const unsigned long long v = S.elems[s];
        const unsigned d = (unsigned)(v >> (32 + shift)) & 0xffu;
        const unsigned long long g = S.gbase[d] + (unsigned long long)(s - (int)S.lbase[d]);
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

size_t hilbert_sort_workspace(int n) {
    if (n <= 0) return 0;
    return sort_layout(nullptr, n).total;
}

tess_status sfc_sort(const float* pos, int n, tess_box box, int bits, int curve, void* ws, size_t ws_bytes,
                     int32_t* perm, uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status, cudaStream_t s) {
    if (n <= 0 || !pos || !perm || !ws || bits < 1 || bits > 10) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (pos_sorted && !aligned(pos_sorted, 16)) return TESS_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return TESS_ERR_INVALID_ARG;
    SortLayout L = sort_layout(ws, n);
    if (ws_bytes < L.total) return TESS_ERR_WORKSPACE_TOO_SMALL;
    int32_t* status = dev_status ? dev_status : L.status;

    cudaMemsetAsync(static_cast<char*>(ws) + L.zero_begin, 0, L.zero_bytes, s);
    if (dev_status) cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s);

    const float g = (float)(1u << bits);
    const float3 scale = make_float3(g / box.lx, g / box.ly, g / box.lz);   // fp32 IEEE divisions
    const int npass = passes_for(bits);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        StageScope sc(ST_KEYS, s);
        const int blocks = (int)std::min<long long>(((long long)n + KEYS_THREADS - 1) / KEYS_THREADS, (long long)sms * 8);
        if (curve == 0)
            keys_kernel<0><<<blocks, KEYS_THREADS, 0, s>>>(pos, n, scale, make_float3(box.lx, box.ly, box.lz), bits,
                                                           npass, L.a, L.hist, status);
        else
            keys_kernel<1><<<blocks, KEYS_THREADS, 0, s>>>(pos, n, scale, make_float3(box.lx, box.ly, box.lz), bits,
                                                           npass, L.a, L.hist, status);
        count_launch();
    }
    {
        StageScope sc(ST_SORT, s);
        const long long tiles = tiles_for(n);
        const size_t smem = sizeof(SortShared);
        static_assert(sizeof(SortShared) <= 48 * 1024, "sort tile must fit the default shared-memory limit");
        unsigned long long* src = L.a;
        unsigned long long* dst = L.b;
        for (int p = 0; p < npass; ++p) {
            unsigned long long* states = L.states + (size_t)p * tiles * RADIX;
            if (p == npass - 1) {
                onesweep_pass<true><<<(unsigned)tiles, SORT_THREADS, smem, s>>>(
                    src, nullptr, n, 8 * p, L.hist + p * RADIX, states, L.counters + p, status, perm, keys_sorted,
                    reinterpret_cast<float4*>(pos_sorted), pos);
            } else {
                onesweep_pass<false><<<(unsigned)tiles, SORT_THREADS, smem, s>>>(
                    src, dst, n, 8 * p, L.hist + p * RADIX, states, L.counters + p, status, nullptr, nullptr,
                    nullptr, nullptr);
            }
            count_launch();
            std::swap(src, dst);
        }
    }
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

}  // namespace tess
