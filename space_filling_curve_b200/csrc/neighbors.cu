// neighbors.cu -- fixed-capacity Verlet list at rs = rc + skin (shapes held
// constant between rebuilds, a neighbor search in three levels; Tessera,
// abstract).
//
// Level 0 (binning, deterministic):
//   cell_count     cell id per atom, warp-aggregated histogram
//   scan_*         exclusive scan of the cell counts -> cell_start
//   cell_scatter   atom indices into their cells (any order within a cell)
//   cell_order     within each cell, order by atom index and write the
//                  positions in cell order as float4 (x, y, z, index bits)
// Levels 1-3 (pair_search, one warp per tile of 32 consecutive atoms, lane =
// atom i):
//   1. tile: bounding box of the 32 atoms (Hilbert-consecutive, so compact)
//   2. cells: every cell row overlapping box +- rs; each cell row is one
//      contiguous range of the cell-ordered positions, shifted by its
//      periodic image; candidates are culled against box +- rs and compacted
//      (ballot + popc) into a shared-memory chunk
//   3. pairs: every lane tests its atom against the chunk (broadcast reads)
//      and appends accepted indices to its row in shared memory; the 32 rows
//      are one contiguous block of the output and leave with 16-byte stores.
#include "common.cuh"

namespace tess {

// ---------------------------------------------------------------- grid

// Cells are at least rs / CELL_DIV wide, so +-CELL_DIV cell rows cover rs.
constexpr int CELL_DIV = 2;

struct Grid {
    int nc[3];
    float inv_w[3];
    long long ncell;
};

// Cells of width about rs/CELL_DIV (the tile search adapts to any width; the
// per-lane stencil relies on width >= rs/CELL_DIV, which coarsening keeps),
// coarsened when that would give more than ~2 cells per atom.
static Grid make_grid(int n, tess_box box, float rs) {
    Grid g{};
    const float L[3] = {box.lx, box.ly, box.lz};
    double w = (double)rs * 1.0001 / (double)CELL_DIV;
    for (int it = 0; it < 64; ++it) {
        long long tot = 1;
        for (int d = 0; d < 3; ++d) {
            long long c = (long long)std::floor((double)L[d] / w);
            if (c < 1) c = 1;
            if (c > (1 << 20)) c = 1 << 20;
            g.nc[d] = (int)c;
            tot *= c;
        }
        g.ncell = tot;
        if (tot <= 2LL * n + 4096) break;
        w *= 1.26;
    }
    for (int d = 0; d < 3; ++d) g.inv_w[d] = (float)g.nc[d] / L[d];   // fp32, shared by all kernels
    return g;
}

__device__ __forceinline__ int cell_coord(float x, float inv_w, int nc) {
    float f = floorf(__fmul_rn(x, inv_w));
    f = fminf(fmaxf(f, 0.0f), (float)(nc - 1));     // NaN -> 0
    return (int)f;
}

// ---------------------------------------------------------------- binning

__global__ void cell_count_kernel(const float4* __restrict__ pos, int n, int3 nc, float3 inv_w, float3 L,
                                  int* __restrict__ cell_id, int* __restrict__ cell_rank, int* __restrict__ cnt,
                                  int32_t* status) {
    bool bad = false;
    const int stride = gridDim.x * blockDim.x;
    for (int base = blockIdx.x * blockDim.x; base < n; base += stride) {
        const int i = base + threadIdx.x;
        const bool valid = i < n;
        int c = -1;
        if (valid) {
            const float4 p = pos[i];
            bad |= !(p.x >= 0.0f && p.x < L.x && p.y >= 0.0f && p.y < L.y && p.z >= 0.0f && p.z < L.z);
            const int cx = cell_coord(p.x, inv_w.x, nc.x);
            const int cy = cell_coord(p.y, inv_w.y, nc.y);
            const int cz = cell_coord(p.z, inv_w.z, nc.z);
            c = (cz * nc.y + cy) * nc.x + cx;
            cell_id[i] = c;
        }
        const unsigned act = __ballot_sync(FULL, valid);
        if (valid) {
            // one atomic per group of lanes in the same cell; each lane keeps its
            // slot among the cell's atoms (any order: cell_order fixes it)
            const unsigned peers = __match_any_sync(act, c);
            const int lane = threadIdx.x & 31, leader = __ffs(peers) - 1;
            int b0 = 0;
            if (lane == leader) b0 = atomicAdd(&cnt[c], __popc(peers));
            b0 = __shfl_sync(peers, b0, leader);
            cell_rank[i] = b0 + __popc(peers & lanemask_lt());
        }
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0 && status) atomicOr(status, TESS_DEV_BAD_INPUT);
}

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

__global__ void cell_scatter_kernel(const int* __restrict__ cell_id, const int* __restrict__ cell_rank, int n,
                                    const int* __restrict__ cell_start, int* __restrict__ slot_atom) {
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        slot_atom[cell_start[cell_id[i]] + cell_rank[i]] = i;
}

// Deterministic order inside each cell: the slot of atom i is the cell start
// plus the number of atoms of the same cell with a smaller index.
__global__ void cell_order_kernel(const int* __restrict__ slot_atom, int n, const int* __restrict__ cell_id,
                                  const int* __restrict__ cell_start, const float4* __restrict__ pos,
                                  float4* __restrict__ pos_cell) {
    const int stride = gridDim.x * blockDim.x;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        const int i = slot_atom[k];
        const int c = cell_id[i];
        const int b = cell_start[c], e = cell_start[c + 1];
        int r = 0;
        for (int s = b; s < e; ++s) r += slot_atom[s] < i;
        const float4 p = pos[i];
        pos_cell[b + r] = make_float4(p.x, p.y, p.z, __int_as_float(i));
    }
}

// ---------------------------------------------------------------- pair search

constexpr int PS_WARPS = 4;          // warps per block (each warp owns its tiles)
constexpr int PS_CHUNK = 256;        // culled candidates staged per warp before testing
constexpr int PS_MAXSEG = 64;        // cell-row segments per table batch
constexpr int PS_UNROLL = 4;         // candidate loads in flight per lane
constexpr int PS_BUF = 32;           // per-lane staging of accepted indices (linear)
constexpr int PS_GROUP = 8;          // accepted indices leave in aligned groups of 8 (32 bytes)
constexpr int PS_TEST_UNROLL = 4;    // candidate pairs tested between fullness votes (the loop is written for 4)

struct PairArgs {
    const float4* pos;
    const float4* pos_cell;
    const int* cell_start;
    int n;
    int cap;
    int pad_fill;
    int vec_rows;      // rows can take 16-byte stores (cap % 4 == 0, 16-byte aligned nbr)
    int3 nc;
    float3 inv_w;
    float3 L;
    float rs2;
    float reach;       // rs plus a margin that covers fp32 rounding of cell and box tests
    int* nbr;
    int* counts;
    int32_t* status;
};

struct SegEntry {
    int beg;
    int pre;           // exclusive prefix of segment lengths within the batch
    float sx, sy, sz, pad0, pad1, pad2;
};

// Per-warp shared memory: candidates as pairs in structure-of-arrays form so
// that one 16-byte read gives (x0, x1, y0, y1) and another (z0, z1, j0, j1),
// ready for packed f32x2 arithmetic; the segment table; the index rings.
struct PairWarpSmem {
    float4 ca[PS_CHUNK / 2];
    float4 cb[PS_CHUNK / 2];
    SegEntry seg[PS_MAXSEG + 1];
    int buf[32 * PS_BUF];
};

__device__ __forceinline__ unsigned long long pk(float lo, float hi) {
    return (unsigned long long)__float_as_uint(lo) | ((unsigned long long)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float pk_lo(unsigned long long v) { return __uint_as_float((unsigned)v); }
__device__ __forceinline__ float pk_hi(unsigned long long v) { return __uint_as_float((unsigned)(v >> 32)); }
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Two 8-byte words from shared memory at base + OFF (OFF an immediate).
template <int OFF>
__device__ __forceinline__ void ld_pair(unsigned base, unsigned long long& a, unsigned long long& b) {
    asm volatile("ld.shared.v2.u64 {%0, %1}, [%2+%3];" : "=l"(a), "=l"(b) : "r"(base), "n"(OFF));
}

// Append candidate j at the buffer slot *wsa and advance the slot by one
// lane-interleaved step (128 bytes) if r2 < rs2 and j is not the atom itself.
// The store happens either way; a rejected index is overwritten by the next.
__device__ __forceinline__ void append_if(unsigned& wsa, float r2, float rs2, int j, int self) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.lt.f32 p, %1, %2;\n\t"
        "setp.ne.and.s32 p, %3, %4, p;\n\t"
        "st.shared.b32 [%0], %3;\n\t"
        "@p add.u32 %0, %0, 128;\n\t}"
        : "+r"(wsa)
        : "f"(r2), "f"(rs2), "r"(j), "r"(self)
        : "memory");
}

// Test one candidate pair (x0,x1), (y0,y1), (z0,z1), (j0,j1) against the atom
// at (px, py, pz) (each duplicated into both halves) with packed f32x2
// arithmetic, and append the accepted indices at *wsa (see append_if).  One
// PTX block, so the halves are never moved out of their register pairs.
__device__ __forceinline__ void test_pair(unsigned& wsa, unsigned long long xx, unsigned long long yy,
                                          unsigned long long zz, unsigned long long jj, unsigned long long px2,
                                          unsigned long long py2, unsigned long long pz2, float rs2, int self) {
    asm volatile(
        "{\n\t.reg .b64 dx, dy, dz, r2;\n\t.reg .f32 r0, r1;\n\t.reg .b32 j0, j1;\n\t.reg .pred p, q;\n\t"
        "sub.rn.f32x2 dx, %1, %5;\n\t"
        "sub.rn.f32x2 dy, %2, %6;\n\t"
        "sub.rn.f32x2 dz, %3, %7;\n\t"
        "mul.rn.f32x2 r2, dx, dx;\n\t"
        "fma.rn.f32x2 r2, dy, dy, r2;\n\t"
        "fma.rn.f32x2 r2, dz, dz, r2;\n\t"
        "mov.b64 {r0, r1}, r2;\n\t"
        "mov.b64 {j0, j1}, %4;\n\t"
        "setp.lt.f32 p, r0, %8;\n\t"
        "setp.ne.and.s32 p, j0, %9, p;\n\t"
        "st.shared.b32 [%0], j0;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "setp.lt.f32 q, r1, %8;\n\t"
        "setp.ne.and.s32 q, j1, %9, q;\n\t"
        "st.shared.b32 [%0], j1;\n\t"
        "@q add.u32 %0, %0, 128;\n\t}"
        : "+r"(wsa)
        : "l"(xx), "l"(yy), "l"(zz), "l"(jj), "l"(px2), "l"(py2), "l"(pz2), "f"(rs2), "r"(self)
        : "memory");
}

// Store one accepted index into slot `slot` of a candidate pair array.
__device__ __forceinline__ void put_cand(PairWarpSmem& W, int slot, float4 q) {
    float* a = reinterpret_cast<float*>(&W.ca[slot >> 1]) + (slot & 1);
    float* b = reinterpret_cast<float*>(&W.cb[slot >> 1]) + (slot & 1);
    a[0] = q.x;
    a[2] = q.y;
    b[0] = q.z;
    b[2] = q.w;
}

__global__ __launch_bounds__(PS_WARPS * 32, 6) void pair_search_kernel(PairArgs A) {
    __shared__ PairWarpSmem smem_w[PS_WARPS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = lanemask_lt();
    PairWarpSmem& W = smem_w[warp];
    // slot s of this lane's buffer is W.buf[s * 32 + lane]: lanes interleaved
    // across the 32 banks, so the appends of a warp never conflict
    int* const buf = W.buf + lane;
    const int cap = A.cap;
    const long long ntiles = ((long long)A.n + 31) / 32;
    const float nanf_ = __int_as_float(0x7fc00000);

    for (long long tile = (long long)blockIdx.x * PS_WARPS + warp; tile < ntiles;
         tile += (long long)gridDim.x * PS_WARPS) {
        const int base = (int)(tile * 32);
        const int i = base + lane;
        const bool valid = i < A.n;
        const float4 p = valid ? A.pos[i] : make_float4(nanf_, nanf_, nanf_, 0.f);
        int* row = A.nbr + (size_t)(valid ? i : 0) * cap;

        // level 1: tile bounding box
        float lox = valid ? p.x : INFINITY, loy = valid ? p.y : INFINITY, loz = valid ? p.z : INFINITY;
        float hix = valid ? p.x : -INFINITY, hiy = valid ? p.y : -INFINITY, hiz = valid ? p.z : -INFINITY;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            lox = fminf(lox, __shfl_xor_sync(FULL, lox, o));
            loy = fminf(loy, __shfl_xor_sync(FULL, loy, o));
            loz = fminf(loz, __shfl_xor_sync(FULL, loz, o));
            hix = fmaxf(hix, __shfl_xor_sync(FULL, hix, o));
            hiy = fmaxf(hiy, __shfl_xor_sync(FULL, hiy, o));
            hiz = fmaxf(hiz, __shfl_xor_sync(FULL, hiz, o));
        }
        // a tile with no finite position (invalid input) searches the whole box;
        // positions far outside the box must not blow up the cell ranges
        if (!(isfinite(lox) && isfinite(hix) && isfinite(loy) && isfinite(hiy) && isfinite(loz) && isfinite(hiz))) {
            lox = loy = loz = 0.f;
            hix = A.L.x; hiy = A.L.y; hiz = A.L.z;
        }
        lox = fmaxf(lox, -A.L.x); loy = fmaxf(loy, -A.L.y); loz = fmaxf(loz, -A.L.z);
        hix = fminf(hix, 2.f * A.L.x); hiy = fminf(hiy, 2.f * A.L.y); hiz = fminf(hiz, 2.f * A.L.z);

        int done = 0;      // accepted indices already written to the row (a multiple of 8 until the end)
        // next free slot of this lane's buffer, as a 32-bit shared-memory address
        const unsigned buf_sa = (unsigned)__cvta_generic_to_shared(buf);
        unsigned wsa = buf_sa;
        int ncand = 0;     // staged candidates (warp-uniform)
        const unsigned long long px2 = pk(p.x, p.x), py2 = pk(p.y, p.y), pz2 = pk(p.z, p.z);
        const float rs2 = A.rs2;

        // write the complete groups of 8 buffered indices to the row; with
        // `all`, the remainder too.  The remainder of a partial drain moves
        // to the front of the buffer.
        auto drain = [&](bool all) {
            const int pend = (int)((wsa - buf_sa) >> 7);
            const int groups = pend / PS_GROUP;
            for (int gi = 0; gi < groups; ++gi) {
                const int* src = buf + gi * PS_GROUP * 32;
                if (done + PS_GROUP <= cap && A.vec_rows) {
                    const int4 a = make_int4(src[0], src[32], src[64], src[96]);
                    const int4 b = make_int4(src[128], src[160], src[192], src[224]);
                    *reinterpret_cast<int4*>(row + done) = a;
                    *reinterpret_cast<int4*>(row + done + 4) = b;
                } else {
                    for (int e = 0; e < PS_GROUP; ++e)
                        if (done + e < cap) row[done + e] = src[e * 32];
                }
                done += PS_GROUP;
            }
            const int rest = pend - groups * PS_GROUP;
            if (all) {
                for (int e = 0; e < rest; ++e)
                    if (done + e < cap) row[done + e] = buf[(groups * PS_GROUP + e) * 32];
                done += rest;
                wsa = buf_sa;
            } else {
                for (int e = 0; e < rest; ++e) buf[e * 32] = buf[(groups * PS_GROUP + e) * 32];
                wsa = buf_sa + 128u * (unsigned)rest;
            }
        };

        // level 3: test the staged candidates, two at a time in f32x2.  An
        // accepted index is stored at the buffer pointer, which then advances
        // (stores for rejected candidates are overwritten by the next one).
        auto test_chunk = [&]() {
            __syncwarp();
            // pad to a whole number of unrolled steps with candidates that are
            // never accepted (NaN position), so the loop needs no bounds tests
            const int padded = (ncand + 2 * PS_TEST_UNROLL - 1) & ~(2 * PS_TEST_UNROLL - 1);
            if (lane < padded - ncand)
                put_cand(W, ncand + lane, make_float4(nanf_, nanf_, nanf_, __int_as_float(-1)));
            __syncwarp();
            const unsigned ca_sa = (unsigned)__cvta_generic_to_shared(&W.ca[0]);
            const unsigned cb_sa = (unsigned)__cvta_generic_to_shared(&W.cb[0]);
            for (int c = 0; c < (padded >> 1); c += PS_TEST_UNROLL) {
                // room for 2 * PS_TEST_UNROLL more in every lane's buffer?
                if (__any_sync(FULL, (int)((wsa - buf_sa) >> 7) > PS_BUF - 2 * PS_TEST_UNROLL)) drain(false);
                unsigned long long xx[4], yy[4], zz[4], jj[4];
                const unsigned ab = ca_sa + 16u * (unsigned)c, bb = cb_sa + 16u * (unsigned)c;
                ld_pair<0>(ab, xx[0], yy[0]);
                ld_pair<0>(bb, zz[0], jj[0]);
                ld_pair<16>(ab, xx[1], yy[1]);
                ld_pair<16>(bb, zz[1], jj[1]);
                ld_pair<32>(ab, xx[2], yy[2]);
                ld_pair<32>(bb, zz[2], jj[2]);
                ld_pair<48>(ab, xx[3], yy[3]);
                ld_pair<48>(bb, zz[3], jj[3]);
#pragma unroll
                for (int u = 0; u < 4; ++u) test_pair(wsa, xx[u], yy[u], zz[u], jj[u], px2, py2, pz2, rs2, i);
            }
            ncand = 0;
            __syncwarp();
        };

        // level 2: cell rows overlapping the box +- reach
        const int ux0 = (int)floorf((lox - A.reach) * A.inv_w.x), ux1 = (int)floorf((hix + A.reach) * A.inv_w.x);
        const int uy0 = (int)floorf((loy - A.reach) * A.inv_w.y), uy1 = (int)floorf((hiy + A.reach) * A.inv_w.y);
        const int uz0 = (int)floorf((loz - A.reach) * A.inv_w.z), uz1 = (int)floorf((hiz + A.reach) * A.inv_w.z);
        const int ny = uy1 - uy0 + 1, nz = uz1 - uz0 + 1;
        const int npieces = floor_div(ux1, A.nc.x) - floor_div(ux0, A.nc.x) + 1;
        const int nseg = ny * nz * npieces;
        const float reach2 = A.reach * A.reach;

        for (int sb = 0; sb < nseg; sb += PS_MAXSEG) {
            const int nb = min(PS_MAXSEG, nseg - sb);
            int run = 0;
            for (int s0 = 0; s0 < nb; s0 += 32) {
                const int sl = s0 + lane;
                int len = 0, beg = 0;
                float sx = 0.f, sy = 0.f, sz = 0.f;
                if (sl < nb) {
                    const int s = sb + sl;
                    const int piece = s % npieces;
                    const int rw = s / npieces;
                    const int uy = uy0 + rw % ny, uz = uz0 + rw / ny;
                    const int ky = floor_div(uy, A.nc.y), kz = floor_div(uz, A.nc.z);
                    const int cy = uy - ky * A.nc.y, cz = uz - kz * A.nc.z;
                    const int kx = floor_div(ux0, A.nc.x) + piece;
                    const int xa = max(ux0, kx * A.nc.x) - kx * A.nc.x;
                    const int xb = min(ux1, (kx + 1) * A.nc.x - 1) - kx * A.nc.x;
                    const int rowbase = (cz * A.nc.y + cy) * A.nc.x;
                    beg = A.cell_start[rowbase + xa];
                    len = A.cell_start[rowbase + xb + 1] - beg;
                    sx = (float)kx * A.L.x;
                    sy = (float)ky * A.L.y;
                    sz = (float)kz * A.L.z;
                }
                int inc = len;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(FULL, inc, o);
                    if (lane >= o) inc += y;
                }
                if (sl < nb) {
                    SegEntry& e = W.seg[sl];
                    e.beg = beg;
                    e.pre = run + inc - len;
                    e.sx = sx; e.sy = sy; e.sz = sz;
                }
                run += __shfl_sync(FULL, inc, 31);
            }
            if (lane == 0) W.seg[nb].pre = run;
            __syncwarp();
            const int total = run;

            int sc = 0;   // this lane's segment cursor
            for (int t0 = 0; t0 < total; t0 += 32 * PS_UNROLL) {
                if (ncand > PS_CHUNK - 2 * PS_TEST_UNROLL - 32 * PS_UNROLL) test_chunk();
                float4 q[PS_UNROLL];
                bool ok[PS_UNROLL];
#pragma unroll
                for (int u = 0; u < PS_UNROLL; ++u) {
                    const int t = t0 + u * 32 + lane;
                    ok[u] = t < total;
                    if (ok[u]) {
                        while (W.seg[sc + 1].pre <= t) ++sc;
                        const SegEntry& e = W.seg[sc];
                        const float4 c = A.pos_cell[e.beg + (t - e.pre)];
                        q[u] = make_float4(c.x + e.sx, c.y + e.sy, c.z + e.sz, c.w);
                    }
                }
#pragma unroll
                for (int u = 0; u < PS_UNROLL; ++u) {
                    bool keep = false;
                    if (ok[u]) {
                        const float ex = fmaxf(fmaxf(lox - q[u].x, q[u].x - hix), 0.f);
                        const float ey = fmaxf(fmaxf(loy - q[u].y, q[u].y - hiy), 0.f);
                        const float ez = fmaxf(fmaxf(loz - q[u].z, q[u].z - hiz), 0.f);
                        keep = fmaf(ez, ez, fmaf(ey, ey, ex * ex)) < reach2;
                    }
                    const unsigned bm = __ballot_sync(FULL, keep);
                    if (keep) put_cand(W, ncand + __popc(bm & lt_mask), q[u]);
                    ncand += __popc(bm);
                }
            }
            __syncwarp();
        }
        test_chunk();
        drain(true);
        const int cnt = done;

        if (valid) {
            A.counts[i] = cnt;
            if (A.pad_fill) {
                int e = min(cnt, cap);
                if (A.vec_rows) {
                    for (; e < cap && (e & 3); ++e) row[e] = -1;
                    for (; e + 4 <= cap; e += 4) *reinterpret_cast<int4*>(row + e) = make_int4(-1, -1, -1, -1);
                }
                for (; e < cap; ++e) row[e] = -1;
            }
        }
        const unsigned ov = __ballot_sync(FULL, valid && cnt > cap);
        if (ov && lane == 0) atomicOr(A.status, TESS_DEV_OVERFLOW);
    }
}

// ---------------------------------------------------------------- per-lane search

// One warp per 32 atoms consecutive in cell order; every lane walks its own stencil:
// the (2 CELL_DIV + 1)^2 cell rows (cells of width >= rs/CELL_DIV, so +-CELL_DIV
// rows cover rs) around
// its own cell, each clipped to the x-window of its own sphere: for a row at
// y/z distance (dy, dz) from the atom the window is x +- sqrt(reach^2 - dy^2 -
// dz^2), and only the cells overlapping it are read.  Candidates are gathered
// per lane (16-byte loads, L1-resident for a compact tile), tested in fp32,
// and accepted indices go through the same bank-interleaved append buffer.
// Loops are warp-uniform (bounded by the warp's longest window) so that the
// buffer vote can run inside them.
constexpr int PL_WARPS = 4;
#ifndef TESS_PL_CHUNK
#define TESS_PL_CHUNK 4
#endif
constexpr int PL_CHUNK = TESS_PL_CHUNK;   // candidates per lane between buffer votes

__global__ __launch_bounds__(PL_WARPS * 32, 6) void pair_search_lane_kernel(PairArgs A) {
    __shared__ int s_buf[PL_WARPS][32 * PS_BUF];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int* const buf = &s_buf[warp][lane];
    const unsigned buf_sa = (unsigned)__cvta_generic_to_shared(buf);
    const int cap = A.cap;
    const long long ntiles = ((long long)A.n + 31) / 32;
    const float wy = (float)A.L.y / (float)A.nc.y, wz = (float)A.L.z / (float)A.nc.z;
    const float reach2 = A.reach * A.reach;
    const float nanf_ = __int_as_float(0x7fc00000);

    for (long long tile = (long long)blockIdx.x * PL_WARPS + warp; tile < ntiles;
         tile += (long long)gridDim.x * PL_WARPS) {
        // lanes take 32 consecutive atoms in cell order (the binning's copy,
        // atom index in w): they share a cell row, so their stencils coincide
        // and their gathers fall on few lines
        const int slot = (int)(tile * 32) + lane;
        const bool valid = slot < A.n;
        const float4 pc = valid ? A.pos_cell[slot] : make_float4(0.f, 0.f, 0.f, 0.f);
        const int i = valid ? __float_as_int(pc.w) : -1;
        float4 p = pc;
        // finite coordinates for the window arithmetic (invalid input is flagged by the binning)
        p.x = fminf(fmaxf(p.x, 0.f), A.L.x);
        p.y = fminf(fmaxf(p.y, 0.f), A.L.y);
        p.z = fminf(fmaxf(p.z, 0.f), A.L.z);
        const float4 p0 = valid ? pc : p;
        int* row = A.nbr + (size_t)(valid ? i : 0) * cap;
        const int cy = cell_coord(p.y, A.inv_w.y, A.nc.y);
        const int cz = cell_coord(p.z, A.inv_w.z, A.nc.z);

        int done = 0;
        unsigned wsa = buf_sa;
        auto drain = [&](bool all) {
            const int pend = (int)((wsa - buf_sa) >> 7);
            const int groups = pend / PS_GROUP;
            for (int gi = 0; gi < groups; ++gi) {
                const int* src = buf + gi * PS_GROUP * 32;
                if (done + PS_GROUP <= cap && A.vec_rows) {
                    const int4 a = make_int4(src[0], src[32], src[64], src[96]);
                    const int4 b = make_int4(src[128], src[160], src[192], src[224]);
                    *reinterpret_cast<int4*>(row + done) = a;
                    *reinterpret_cast<int4*>(row + done + 4) = b;
                } else {
                    for (int e = 0; e < PS_GROUP; ++e)
                        if (done + e < cap) row[done + e] = src[e * 32];
                }
                done += PS_GROUP;
            }
            const int rest = pend - groups * PS_GROUP;
            if (all) {
                for (int e = 0; e < rest; ++e)
                    if (done + e < cap) row[done + e] = buf[(groups * PS_GROUP + e) * 32];
                done += rest;
                wsa = buf_sa;
            } else {
                for (int e = 0; e < rest; ++e) buf[e * 32] = buf[(groups * PS_GROUP + e) * 32];
                wsa = buf_sa + 128u * (unsigned)rest;
            }
        };

        float4 c[PL_CHUNK];
#pragma unroll
        for (int u = 0; u < PL_CHUNK; ++u) c[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int dz = -CELL_DIV; dz <= CELL_DIV; ++dz) {
            // row z: unwrapped index for the geometry, wrapped index and image shift for the data
            int wz_i = cz + dz, kz = 0;
            while (wz_i < 0) { wz_i += A.nc.z; --kz; }
            while (wz_i >= A.nc.z) { wz_i -= A.nc.z; ++kz; }
            const float zlo = (float)(cz + dz) * wz;
            const float ddz = fmaxf(fmaxf(zlo - p.z, p.z - (zlo + wz)), 0.f);
            const float qz = p0.z - (float)kz * A.L.z;
            for (int dy = -CELL_DIV; dy <= CELL_DIV; ++dy) {
                int wy_i = cy + dy, ky = 0;
                while (wy_i < 0) { wy_i += A.nc.y; --ky; }
                while (wy_i >= A.nc.y) { wy_i -= A.nc.y; ++ky; }
                const float ylo = (float)(cy + dy) * wy;
                const float ddy = fmaxf(fmaxf(ylo - p.y, p.y - (ylo + wy)), 0.f);
                const float ch2 = reach2 - ddy * ddy - ddz * ddz;
                const float qy = p0.y - (float)ky * A.L.y;
                int beg[2] = {0, 0}, len[2] = {0, 0};
                float qx[2] = {0.f, 0.f};
                if (valid && ch2 > 0.f) {
                    // x-chord of the sphere in this row (approximate root, widened)
                    const float chord = fmaf(ch2 * rsqrtf(ch2), 1.0001f, 1e-4f);
                    const int rowbase = (wz_i * A.nc.y + wy_i) * A.nc.x;
                    int ua = (int)floorf((p.x - chord) * A.inv_w.x);
                    int ub = (int)floorf((p.x + chord) * A.inv_w.x);
                    int kx = 0;
                    while (ua < 0) { ua += A.nc.x; ub += A.nc.x; --kx; }
                    while (ua >= A.nc.x) { ua -= A.nc.x; ub -= A.nc.x; ++kx; }
                    // with L >= 2 reach the window covers at most nc.x + 1
                    // cells, so it wraps at most once: two contiguous pieces
                    const int e0 = min(ub, A.nc.x - 1);
                    beg[0] = A.cell_start[rowbase + ua];
                    len[0] = A.cell_start[rowbase + e0 + 1] - beg[0];
                    qx[0] = p0.x - (float)kx * A.L.x;
                    if (ub >= A.nc.x) {
                        const int e1 = min(ub - A.nc.x, A.nc.x - 1);
                        beg[1] = A.cell_start[rowbase];
                        len[1] = A.cell_start[rowbase + e1 + 1] - beg[1];
                        qx[1] = p0.x - (float)(kx + 1) * A.L.x;
                    }
                }
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const int maxlen = (int)__reduce_max_sync(FULL, (unsigned)len[pc]);
                    for (int k0 = 0; k0 < maxlen; k0 += PL_CHUNK) {
                        if (__any_sync(FULL, (int)((wsa - buf_sa) >> 7) > PS_BUF - PL_CHUNK)) drain(false);
                        // slots past this lane's window keep stale data; their
                        // index becomes the atom's own, which the test rejects, so
                        // the test below needs no branch
                        const float4* src = A.pos_cell + beg[pc] + k0;
#pragma unroll
                        for (int u = 0; u < PL_CHUNK; ++u)
                            if (k0 + u < len[pc]) c[u] = src[u];
#pragma unroll
                        for (int u = 0; u < PL_CHUNK; ++u) {
                            const float dx = c[u].x - qx[pc];
                            const float ddy2 = c[u].y - qy;
                            const float ddz2 = c[u].z - qz;
                            const float r2 = fmaf(ddz2, ddz2, fmaf(ddy2, ddy2, dx * dx));
                            append_if(wsa, r2, A.rs2, (k0 + u < len[pc]) ? __float_as_int(c[u].w) : i, i);
                        }
                    }
                }
            }
        }
        drain(true);
        const int cnt = done;
        if (valid) {
            A.counts[i] = cnt;
            if (A.pad_fill) {
                int e = min(cnt, cap);
                if (A.vec_rows) {
                    for (; e < cap && (e & 3); ++e) row[e] = -1;
                    for (; e + 4 <= cap; e += 4) *reinterpret_cast<int4*>(row + e) = make_int4(-1, -1, -1, -1);
                }
                for (; e < cap; ++e) row[e] = -1;
            }
        }
        const unsigned ov = __ballot_sync(FULL, valid && cnt > cap);
        if (ov && lane == 0) atomicOr(A.status, TESS_DEV_OVERFLOW);
    }
}

// ---------------------------------------------------------------- host

struct NbrLayout {
    int* cell_id;
    int* cell_rank;
    int* cnt;
    int* cell_start;
    int* sums;
    int* slot_atom;
    float4* pos_cell;
    int32_t* status;
    size_t total;
};

static NbrLayout nbr_layout(void* ws, int n, const Grid& g) {
    Carve c(ws);
    NbrLayout L{};
    const long long m = g.ncell;
    L.cell_id = c.take<int>((size_t)n);
    L.cell_rank = c.take<int>((size_t)n);
    L.cnt = c.take<int>((size_t)m);
    L.cell_start = c.take<int>((size_t)m + 1);
    L.sums = c.take<int>((size_t)((m + SCAN_TILE - 1) / SCAN_TILE) + 1);
    L.slot_atom = c.take<int>((size_t)n);
    L.pos_cell = c.take<float4>((size_t)n);
    L.status = c.take<int32_t>(1);
    L.total = align_up(c.off, 256);
    return L;
}

static bool box_ok(tess_box b) { return finite_pos(b.lx) && finite_pos(b.ly) && finite_pos(b.lz); }

size_t build_neighbors_workspace(int n, tess_box box, float rc, float skin) {
    if (n <= 0 || !box_ok(box) || !(rc > 0.f) || !(skin >= 0.f)) return 0;
    const float rs = rc + skin;
    return nbr_layout(nullptr, n, make_grid(n, box, rs)).total;
}

tess_status build_neighbors(const float* pos, int n, tess_box box, float rc, float skin, int cap, int flags,
                            void* ws, size_t ws_bytes, int32_t* nbr, int32_t* counts, int32_t* overflow,
                            cudaStream_t s) {
    if (n <= 0 || !pos || !ws || !nbr || !counts || !overflow || cap < 1) return TESS_ERR_INVALID_ARG;
    if (!box_ok(box) || !(rc > 0.f) || !(skin >= 0.f) || !std::isfinite(rc) || !std::isfinite(skin))
        return TESS_ERR_INVALID_ARG;
    if ((flags & ~(TESS_NO_PAD_FILL | TESS_TILE_SEARCH)) != 0) return TESS_ERR_INVALID_ARG;
    if (!aligned(pos, 16) || !aligned(ws, 256) || !aligned(nbr, 4) || !aligned(counts, 4)) return TESS_ERR_INVALID_ARG;
    const float rs = rc + skin;
    if (box.lx < 2.f * rs || box.ly < 2.f * rs || box.lz < 2.f * rs) return TESS_ERR_BOX_TOO_SMALL;
    const Grid g = make_grid(n, box, rs);
    NbrLayout L = nbr_layout(ws, n, g);
    if (ws_bytes < L.total) return TESS_ERR_WORKSPACE_TOO_SMALL;

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const float4* pos4 = reinterpret_cast<const float4*>(pos);
    const int3 nc = make_int3(g.nc[0], g.nc[1], g.nc[2]);
    const float3 inv_w = make_float3(g.inv_w[0], g.inv_w[1], g.inv_w[2]);
    const float3 Lb = make_float3(box.lx, box.ly, box.lz);
    const long long m = g.ncell;
    const long long scan_tiles = (m + SCAN_TILE - 1) / SCAN_TILE;

    cudaMemsetAsync(overflow, 0, sizeof(int32_t), s);
    {
        StageScope sc(ST_CELLS, s);
        cudaMemsetAsync(L.cnt, 0, sizeof(int) * (size_t)m, s);
        const int blocks = (int)std::min<long long>(((long long)n + 255) / 256, (long long)sms * 16);
        cell_count_kernel<<<blocks, 256, 0, s>>>(pos4, n, nc, inv_w, Lb, L.cell_id, L.cell_rank, L.cnt, overflow);
        scan_reduce_kernel<<<(unsigned)scan_tiles, SCAN_THREADS, 0, s>>>(L.cnt, m, L.sums);
        scan_sums_kernel<<<1, SCAN_THREADS, 0, s>>>(L.sums, scan_tiles);
        scan_apply_kernel<<<(unsigned)scan_tiles, SCAN_THREADS, 0, s>>>(L.cnt, m, L.sums, L.cell_start);
        cell_scatter_kernel<<<blocks, 256, 0, s>>>(L.cell_id, L.cell_rank, n, L.cell_start, L.slot_atom);
        cell_order_kernel<<<blocks, 256, 0, s>>>(L.slot_atom, n, L.cell_id, L.cell_start, pos4, L.pos_cell);
        count_launch(6);
    }
    {
        StageScope sc(ST_PAIRS, s);
        PairArgs A;
        A.pos = pos4;
        A.pos_cell = L.pos_cell;
        A.cell_start = L.cell_start;
        A.n = n;
        A.cap = cap;
        A.pad_fill = (flags & TESS_NO_PAD_FILL) ? 0 : 1;
        A.vec_rows = (cap % 4 == 0 && aligned(nbr, 16)) ? 1 : 0;
        A.nc = nc;
        A.inv_w = inv_w;
        A.L = Lb;
        A.rs2 = rs * rs;
        const float lmax = std::max(box.lx, std::max(box.ly, box.lz));
        A.reach = rs + 1e-3f + 4e-6f * lmax;
        A.nbr = nbr;
        A.counts = counts;
        A.status = overflow;
        const long long ntiles = ((long long)n + 31) / 32;
        // the per-lane search needs every box length >= 2 reach (a window
        // then wraps at most once); otherwise the tile search handles it
        const bool lane_ok = box.lx >= 2.f * A.reach && box.ly >= 2.f * A.reach && box.lz >= 2.f * A.reach;
        if ((flags & TESS_TILE_SEARCH) || !lane_ok) {
            const long long blocks = (ntiles + PS_WARPS - 1) / PS_WARPS;
            pair_search_kernel<<<(unsigned)std::min<long long>(blocks, 1LL << 30), PS_WARPS * 32, 0, s>>>(A);
        } else {
            const long long blocks = (ntiles + PL_WARPS - 1) / PL_WARPS;
            pair_search_lane_kernel<<<(unsigned)std::min<long long>(blocks, 1LL << 30), PL_WARPS * 32, 0, s>>>(A);
        }
        count_launch();
    }
    return launch_status();
}

}  // namespace tess
