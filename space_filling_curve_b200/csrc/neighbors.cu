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
// Levels 1-3 (pair_tile_kernel, the default; one warp per tile of 32
// consecutive atoms, lane = atom i):
//   1. tile: bounding box of the 32 atoms (Hilbert-consecutive, so compact)
//      and a frame centred on it
//   2. cells: the cell rows within reach of the box, each clipped to the
//      box's chord at its distance; each piece of a row is one contiguous
//      range of the cell-ordered positions, shifted by its periodic image;
//      candidates are culled against the rounded box and compacted (ballot
//      + popc) into a shared-memory chunk
//   3. pairs: every lane tests its atom against the chunk (broadcast reads,
//      packed f32x2), 32 candidates per accept mask, and turns the set bits
//      into indices that leave for its row in aligned 32-byte groups.
// pair_search_lane_kernel (TESS_LANE_SEARCH) walks a stencil of cell rows
// per lane instead; it gives the same lists in another order.  Which of the
// two runs when the caller asks for neither is TESS_DEFAULT_LANE.
#include <climits>

#include "common.cuh"
#include "scan.cuh"

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

__global__ void cell_scatter_kernel(const int* __restrict__ cell_id, const int* __restrict__ cell_rank, int n,
                                    const int* __restrict__ cell_start, int* __restrict__ slot_atom,
                                    int32_t* status) {
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const long long slot = (long long)cell_start[cell_id[i]] + cell_rank[i];
        if (check_index(slot, n, status)) slot_atom[slot] = i;
    }
}

// Deterministic order inside each cell: the atoms of a cell in ascending
// index order, positions written in that order as float4 (x, y, z, index
// bits).  One thread per cell; cells of up to 8 atoms (nearly all) are sorted
// in registers by a fixed network, larger ones rank each atom by counting.
__device__ __forceinline__ void cswap(int& a, int& b) {
    const int lo = min(a, b), hi = max(a, b);
    a = lo;
    b = hi;
}

__global__ void cell_order_kernel(const int* __restrict__ slot_atom, long long ncell,
                                  const int* __restrict__ cell_start, const float4* __restrict__ pos,
                                  float4* __restrict__ pos_cell) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < ncell; c += stride) {
        const int b = cell_start[c], e = cell_start[c + 1], m = e - b;
        if (m <= 0) continue;
        if (m <= 8) {
            int v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = k < m ? slot_atom[b + k] : INT_MAX;
            // Batcher's odd-even merge network for 8 (19 comparators)
            cswap(v[0], v[1]); cswap(v[2], v[3]); cswap(v[4], v[5]); cswap(v[6], v[7]);
            cswap(v[0], v[2]); cswap(v[1], v[3]); cswap(v[4], v[6]); cswap(v[5], v[7]);
            cswap(v[1], v[2]); cswap(v[5], v[6]);
            cswap(v[0], v[4]); cswap(v[1], v[5]); cswap(v[2], v[6]); cswap(v[3], v[7]);
            cswap(v[2], v[4]); cswap(v[3], v[5]);
            cswap(v[1], v[2]); cswap(v[3], v[4]); cswap(v[5], v[6]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (k < m) {
                    const float4 p = pos[v[k]];
                    pos_cell[b + k] = make_float4(p.x, p.y, p.z, __int_as_float(v[k]));
                }
            }
        } else {
            for (int s = b; s < e; ++s) {
                const int i = slot_atom[s];
                int r = 0;
                for (int t = b; t < e; ++t) r += slot_atom[t] < i;
                const float4 p = pos[i];
                pos_cell[b + r] = make_float4(p.x, p.y, p.z, __int_as_float(i));
            }
        }
    }
}

// ---------------------------------------------------------------- pair search

constexpr int PS_BUF = 32;           // per-lane staging of accepted indices, per-lane search
constexpr int PS_GROUP = 8;          // accepted indices leave in aligned groups of 8 (32 bytes)

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

// ------------------------------------------------ tile search with accept masks
//
// One warp per tile of 32 consecutive atoms (Hilbert-consecutive when the
// input is sorted, so the tile is compact), lane = atom i.
//   1. tile frame: bounding box of the 32 atoms (shuffles) and its centre o;
//      every coordinate below is taken relative to o, so the pair test works
//      on numbers of a few Angstrom.
//   2. candidates: the cell rows within reach of the box, each row clipped to
//      the chord of the rounded box at that row's y/z distance; every atom
//      read is culled against the rounded box (distance to the box < reach)
//      and the survivors are compacted (ballot + popc) into a shared-memory
//      chunk in groups of four: x0 x1 y0 y1 | z0 z1 x2 x3 | y2 y3 z2 z3, so
//      that three broadcast 16-byte reads feed packed f32x2 arithmetic for
//      four candidates.
//   3. pairs: per block of 32 staged candidates every lane builds a 32-bit
//      accept mask (r^2 < rs^2), then walks its set bits, skipping itself,
//      into a lane-interleaved buffer that drains to the row in aligned
//      32-byte groups.  Pads follow as coalesced stores, row by row.

constexpr int TM_WARPS = 4;          // warps per block, each on its own tiles
constexpr int TM_CH = 256;           // staged candidates per chunk (a multiple of 32)
constexpr int TM_MAXSEG = 64;        // cell-row segments per table batch
#ifndef TESS_TM_RANGES
#define TESS_TM_RANGES 0
#endif
#ifndef TESS_TM_UNROLL
#define TESS_TM_UNROLL 4
#endif
constexpr int TM_UNROLL = TESS_TM_UNROLL;  // candidate loads in flight per lane while culling
constexpr int TM_BUF = 48;           // per-lane buffer of accepted indices (>= 32 + TM_GROUP)
constexpr int TM_GROUP = 8;          // indices leave in aligned groups of 8 (32 bytes)
constexpr float TM_FFMA_H = 12.f;    // largest tile half-diagonal (A) for the fused pair test

struct TileWarpSmem {
    float cq[TM_CH * 4];             // staged candidates, 64 bytes per group of four (tile frame)
    int cj[TM_CH];                   // their atom indices
    SegEntry seg[TM_MAXSEG + 1];
    int buf[32 * TM_BUF];            // entry e of lane l at buf[e * 32 + l]
};
constexpr size_t TM_SMEM = sizeof(TileWarpSmem) * TM_WARPS;

// Candidate s of the chunk: group s / 4 holds x0 x1 y0 y1 | z0 z1 n0 n1 |
// x2 x3 y2 y3 | z2 z3 n2 n3 (tile frame, n = x^2 + y^2 + z^2), so that each
// 16-byte read gives two candidates' values of one kind, ready for packed
// f32x2 arithmetic.
__device__ __forceinline__ void stage_cand(TileWarpSmem& W, int s, float x, float y, float z, int j) {
    const int k = s & 3;
    const int off = 16 * (s >> 2) + (k & 1) + (k >> 1) * 8;
    W.cq[off] = x;
    W.cq[off + 2] = y;
    W.cq[off + 4] = z;
    W.cq[off + 6] = fmaf(z, z, fmaf(y, y, x * x));
    W.cj[s] = j;
}

// Both pair tests below append each accepted index to the lane's buffer: it
// is stored at the lane's next slot (*wsa) and the slot advances by one
// lane-interleaved step (128 bytes).

// Compact tiles: r^2 < rs^2  <=>  |c|^2 - 2 c.p < rs^2 - |p|^2 = T in the tile
// frame (|c|, |p| of a few Angstrom), three packed fused multiply-adds per
// two candidates: v = n + c.m with m = -2 p (m2x, m2y, m2z in both halves).
// The tile's own atoms are not among the candidates (they are tested by
// intra_tile), so no index comparison is needed.
template <int G>
__device__ __forceinline__ void test4_ffma(unsigned& wsa, const ulonglong2* q, const int4* qj,
                                           unsigned long long m2x, unsigned long long m2y,
                                           unsigned long long m2z, float T) {
    const ulonglong2 a = q[4 * G], b = q[4 * G + 1], c = q[4 * G + 2], d = q[4 * G + 3];
    const int4 j = qj[G];
    asm volatile(
        "{\n\t.reg .b64 v;\n\t.reg .f32 v0, v1;\n\t.reg .pred p;\n\t"
        "fma.rn.f32x2 v, %1, %9, %4;\n\t"
        "fma.rn.f32x2 v, %2, %10, v;\n\t"
        "fma.rn.f32x2 v, %3, %11, v;\n\t"
        "mov.b64 {v0, v1}, v;\n\t"
        "setp.lt.f32 p, v0, %12;\n\t"
        "@p st.shared.b32 [%0], %13;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "setp.lt.f32 p, v1, %12;\n\t"
        "@p st.shared.b32 [%0], %14;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "fma.rn.f32x2 v, %5, %9, %8;\n\t"
        "fma.rn.f32x2 v, %6, %10, v;\n\t"
        "fma.rn.f32x2 v, %7, %11, v;\n\t"
        "mov.b64 {v0, v1}, v;\n\t"
        "setp.lt.f32 p, v0, %12;\n\t"
        "@p st.shared.b32 [%0], %15;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "setp.lt.f32 p, v1, %12;\n\t"
        "@p st.shared.b32 [%0], %16;\n\t"
        "@p add.u32 %0, %0, 128;\n\t}"
        : "+r"(wsa)
        : "l"(a.x), "l"(a.y), "l"(b.x), "l"(b.y), "l"(c.x), "l"(c.y), "l"(d.x), "l"(d.y), "l"(m2x), "l"(m2y),
          "l"(m2z), "f"(T), "r"(j.x), "r"(j.y), "r"(j.z), "r"(j.w)
        : "memory");
}

// Any tile: differences (x, y, z of candidate minus atom, both in the tile
// frame), r^2 = (dx^2 + dy^2) + dz^2 with packed arithmetic, r^2 < rs^2, and
// the atom itself (index `self`) skipped.
template <int G>
__device__ __forceinline__ void test4_sub(unsigned& wsa, const ulonglong2* q, const int4* qj,
                                          unsigned long long px2, unsigned long long py2,
                                          unsigned long long pz2, float rs2, int self) {
    const ulonglong2 a = q[4 * G], b = q[4 * G + 1], c = q[4 * G + 2], d = q[4 * G + 3];
    const int4 j = qj[G];
    asm volatile(
        "{\n\t.reg .b64 dx, dy, dz, r;\n\t.reg .f32 r0, r1;\n\t.reg .pred p;\n\t"
        "sub.rn.f32x2 dx, %1, %7;\n\t"
        "sub.rn.f32x2 dy, %2, %8;\n\t"
        "sub.rn.f32x2 dz, %3, %9;\n\t"
        "mul.rn.f32x2 r, dx, dx;\n\t"
        "fma.rn.f32x2 r, dy, dy, r;\n\t"
        "fma.rn.f32x2 r, dz, dz, r;\n\t"
        "mov.b64 {r0, r1}, r;\n\t"
        "setp.lt.f32 p, r0, %10;\n\t"
        "setp.ne.and.s32 p, %11, %15, p;\n\t"
        "@p st.shared.b32 [%0], %11;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "setp.lt.f32 p, r1, %10;\n\t"
        "setp.ne.and.s32 p, %12, %15, p;\n\t"
        "@p st.shared.b32 [%0], %12;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "sub.rn.f32x2 dx, %4, %7;\n\t"
        "sub.rn.f32x2 dy, %5, %8;\n\t"
        "sub.rn.f32x2 dz, %6, %9;\n\t"
        "mul.rn.f32x2 r, dx, dx;\n\t"
        "fma.rn.f32x2 r, dy, dy, r;\n\t"
        "fma.rn.f32x2 r, dz, dz, r;\n\t"
        "mov.b64 {r0, r1}, r;\n\t"
        "setp.lt.f32 p, r0, %10;\n\t"
        "setp.ne.and.s32 p, %13, %15, p;\n\t"
        "@p st.shared.b32 [%0], %13;\n\t"
        "@p add.u32 %0, %0, 128;\n\t"
        "setp.lt.f32 p, r1, %10;\n\t"
        "setp.ne.and.s32 p, %14, %15, p;\n\t"
        "@p st.shared.b32 [%0], %14;\n\t"
        "@p add.u32 %0, %0, 128;\n\t}"
        : "+r"(wsa)
        : "l"(a.x), "l"(a.y), "l"(b.x), "l"(c.x), "l"(c.y), "l"(d.x), "l"(px2), "l"(py2), "l"(pz2), "f"(rs2),
          "r"(j.x), "r"(j.y), "r"(j.z), "r"(j.w), "r"(self)
        : "memory");
}

// q = a / b, r = a % b for 0 <= a < 2^22 and a small divisor b > 0, through
// the fp32 reciprocal and one correction step (cheaper than integer division).
__device__ __forceinline__ void div_small(int a, int b, float inv_b, int& q, int& r) {
    q = (int)((float)a * inv_b);
    r = a - q * b;
    if (r < 0) { --q; r += b; }
    else if (r >= b) { ++q; r -= b; }
}

__device__ __forceinline__ unsigned long long pk2(float v) {
    return (unsigned long long)__float_as_uint(v) | ((unsigned long long)__float_as_uint(v) << 32);
}

// The list is written once and read by later kernels; its stores are marked
// streaming (evict first) so that they do not push the candidate positions,
// which every tile reads again, out of L2.
#ifndef TESS_TM_CS
#define TESS_TM_CS 1
#endif
#if TESS_TM_CS
#define TESS_ST_COP ".cs"
#else
#define TESS_ST_COP ""
#endif

// Eight consecutive ints to a 32-byte aligned global address.
__device__ __forceinline__ void st_global_v8(int* p, int a0, int a1, int a2, int a3, int a4, int a5, int a6, int a7) {
    asm volatile("st.global" TESS_ST_COP ".v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0),
                 "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
                 : "memory");
}
// Four consecutive ints to a 16-byte aligned global address.
__device__ __forceinline__ void st_global_v4(int* p, int a0, int a1, int a2, int a3) {
    asm volatile("st.global" TESS_ST_COP ".v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
                 "r"(a3)
                 : "memory");
}

// VW: row store width in ints (8: rows 32-byte aligned, cap % 8 == 0;
// 4: 16-byte aligned, cap % 4 == 0; 1: anything).
template <int VW>
__global__ __launch_bounds__(TM_WARPS * 32, 4) void pair_tile_kernel(PairArgs A) {
    extern __shared__ __align__(16) unsigned char tm_smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt_mask = lanemask_lt();
    TileWarpSmem& W = reinterpret_cast<TileWarpSmem*>(tm_smem_raw)[warp];
    int* const buf = W.buf + lane;
    const unsigned buf_sa = (unsigned)__cvta_generic_to_shared(buf);
    const int cap = A.cap;
    const long long ntiles = ((long long)A.n + 31) / 32;
    const float nanf_ = __int_as_float(0x7fc00000);
    const float wy = A.L.y / (float)A.nc.y, wz = A.L.z / (float)A.nc.z;
    const float reach2 = A.reach * A.reach;

#if TESS_TM_RANGES
    // each block walks its own contiguous range of tiles (its warps side by
    // side), so that an SM works on neighboring tiles whose candidate cells
    // overlap and stay in its L1
    const long long per_block = (ntiles + gridDim.x - 1) / gridDim.x;
    const long long t_end = min(ntiles, (long long)(blockIdx.x + 1) * per_block);
    for (long long tile = (long long)blockIdx.x * per_block + warp; tile < t_end; tile += TM_WARPS) {
#else
    for (long long tile = (long long)blockIdx.x * TM_WARPS + warp; tile < ntiles;
         tile += (long long)gridDim.x * TM_WARPS) {
#endif
        const int base = (int)(tile * 32);
        const int i = base + lane;
        const bool valid = i < A.n;
        const float4 p = valid ? A.pos[i] : make_float4(nanf_, nanf_, nanf_, 0.f);
        int* const row = A.nbr + (size_t)(valid ? i : 0) * cap;

        // level 1: tile bounding box and frame
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
        const float ox = 0.5f * (lox + hix), oy = 0.5f * (loy + hiy), oz = 0.5f * (loz + hiz);
        const float qx = p.x - ox, qy = p.y - oy, qz = p.z - oz;     // the atom in the tile frame
        const unsigned long long px2 = pk2(qx), py2 = pk2(qy), pz2 = pk2(qz);
        const float rs2 = A.rs2;
        // A compact tile (the usual case) uses the fused form of the pair
        // test, whose fp32 error grows with the frame's size: for a
        // half-diagonal up to TM_FFMA_H the terms stay below ~800 A^2 and the
        // rounding of n, T and the three products moves r^2 by at most
        // ~1.6e-4 A^2, about 1.3e-5 A in r near rs -- well inside the 1e-4 A
        // band that the inputs keep around rs.  It also leaves its own atoms
        // out of the candidates: they are tested against each other directly,
        // which needs every pair inside the tile to be its own minimum image.
        const float hx = 0.5f * (hix - lox), hy = 0.5f * (hiy - loy), hz = 0.5f * (hiz - loz);
        const bool compact = fmaf(hz, hz, fmaf(hy, hy, hx * hx)) <= TM_FFMA_H * TM_FFMA_H &&
                             4.f * hx < A.L.x - 2.f * A.reach && 4.f * hy < A.L.y - 2.f * A.reach &&
                             4.f * hz < A.L.z - 2.f * A.reach;
        const unsigned long long m2x = pk2(-2.f * qx), m2y = pk2(-2.f * qy), m2z = pk2(-2.f * qz);
        const float T = rs2 - fmaf(qz, qz, fmaf(qy, qy, qx * qx));

        int done = 0;      // accepted indices handed to the row (a multiple of TM_GROUP until the end)
        int pend = 0;      // indices waiting in this lane's buffer
        int ncand = 0;     // staged candidates (warp-uniform)

        // write the complete groups of TM_GROUP buffered indices to the row;
        // the rest moves to the front of the buffer
        auto drain = [&]() {
            const int groups = pend / TM_GROUP;
            for (int gi = 0; gi < groups; ++gi) {
                const int* src = buf + gi * TM_GROUP * 32;
                if (VW == 8 && done + TM_GROUP <= cap) {
                    st_global_v8(row + done, src[0], src[32], src[64], src[96], src[128], src[160], src[192],
                                 src[224]);
                } else if (VW == 4 && done + TM_GROUP <= cap) {
                    st_global_v4(row + done, src[0], src[32], src[64], src[96]);
                    st_global_v4(row + done + 4, src[128], src[160], src[192], src[224]);
                } else {
#pragma unroll
                    for (int e = 0; e < TM_GROUP; ++e)
                        if (done + e < cap) row[done + e] = src[e * 32];
                }
                done += TM_GROUP;
            }
            const int rest = pend - groups * TM_GROUP;
            for (int e = 0; e < rest; ++e) buf[e * 32] = buf[(groups * TM_GROUP + e) * 32];
            pend = rest;
        };

        // level 3: test the staged candidates in blocks of 32.  With `last`
        // the final partial block is padded with candidates that are never
        // accepted (NaN); otherwise it moves to the front of the chunk.
        auto test_chunk = [&](bool last) {
            __syncwarp();
            int nblk = ncand >> 5;
            if (last && (ncand & 31)) {
                const int pad_to = (ncand + 31) & ~31;
                if (lane < pad_to - ncand) stage_cand(W, ncand + lane, nanf_, nanf_, nanf_, -1);
                nblk = pad_to >> 5;
                __syncwarp();
            }
            for (int blk = 0; blk < nblk; ++blk) {
                if (__any_sync(FULL, pend > TM_BUF - 32)) drain();
                const ulonglong2* q = reinterpret_cast<const ulonglong2*>(W.cq + blk * 128);
                const int4* qj = reinterpret_cast<const int4*>(W.cj + blk * 32);
                unsigned wsa = buf_sa + 128u * (unsigned)pend;
                if (compact) {
                    test4_ffma<0>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<1>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<2>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<3>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<4>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<5>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<6>(wsa, q, qj, m2x, m2y, m2z, T);
                    test4_ffma<7>(wsa, q, qj, m2x, m2y, m2z, T);
                } else {
                    test4_sub<0>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<1>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<2>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<3>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<4>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<5>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<6>(wsa, q, qj, px2, py2, pz2, rs2, i);
                    test4_sub<7>(wsa, q, qj, px2, py2, pz2, rs2, i);
                }
                pend = (int)((wsa - buf_sa) >> 7);
            }
            if (last) {
                ncand = 0;
            } else {
                // the partial block (fewer than 32) moves to the front: whole
                // 64-byte groups and their indices
                const int rem = ncand - (nblk << 5);
                __syncwarp();
                float4* cq4 = reinterpret_cast<float4*>(W.cq);
                const int nq = ((rem + 3) >> 2) * 4;
                float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
                int tj = 0;
                if (lane < nq) t4 = cq4[nblk * 32 + lane];
                if (lane < rem) tj = W.cj[(nblk << 5) + lane];
                __syncwarp();
                if (lane < nq) cq4[lane] = t4;
                if (lane < rem) W.cj[lane] = tj;
                ncand = rem;
            }
            __syncwarp();
        };

        // the tile's own atoms against each other (compact tiles): the other
        // 31 lanes' frame coordinates by shuffles, the same fp32 difference
        // form as test4_sub; its indices enter the (empty) buffer first
        if (compact) {
            unsigned wsa = buf_sa;
            for (int o = 1; o < 32; ++o) {
                const int src = (lane + o) & 31;
                const float dx = __shfl_sync(FULL, qx, src) - qx;
                const float dy = __shfl_sync(FULL, qy, src) - qy;
                const float dz = __shfl_sync(FULL, qz, src) - qz;
                const float r2 = fmaf(dz, dz, fmaf(dy, dy, dx * dx));
                append_if(wsa, r2, rs2, base + src, i);
            }
            pend = (int)((wsa - buf_sa) >> 7);
        }

        // level 2: cell rows within reach of the box, each clipped to its chord
        const int ux0 = (int)floorf((lox - A.reach) * A.inv_w.x), ux1 = (int)floorf((hix + A.reach) * A.inv_w.x);
        const int uy0 = (int)floorf((loy - A.reach) * A.inv_w.y), uy1 = (int)floorf((hiy + A.reach) * A.inv_w.y);
        const int uz0 = (int)floorf((loz - A.reach) * A.inv_w.z), uz1 = (int)floorf((hiz + A.reach) * A.inv_w.z);
        const int ny = uy1 - uy0 + 1, nz = uz1 - uz0 + 1;
        const int kx0 = floor_div(ux0, A.nc.x);
        const int npieces = floor_div(ux1, A.nc.x) - kx0 + 1;
        const int nseg = ny * nz * npieces;
        const float inv_np = 1.0f / (float)npieces, inv_ny = 1.0f / (float)ny;

        for (int sb = 0; sb < nseg; sb += TM_MAXSEG) {
            const int nb = min(TM_MAXSEG, nseg - sb);
            int run = 0;
            for (int s0 = 0; s0 < nb; s0 += 32) {
                const int sl = s0 + lane;
                int len = 0, beg = 0;
                float sx = 0.f, sy = 0.f, sz = 0.f;
                if (sl < nb) {
                    const int s = sb + sl;
                    // s = rw * npieces + piece, rw = (uz - uz0) * ny + (uy - uy0)
                    int rw, piece, rz, ry;
                    div_small(s, npieces, inv_np, rw, piece);
                    div_small(rw, ny, inv_ny, rz, ry);
                    const int uy = uy0 + ry, uz = uz0 + rz;
                    // the row's distance to the box in y and z (unwrapped cell geometry)
                    const float ylo = (float)uy * wy, zlo = (float)uz * wz;
                    const float ddy = fmaxf(fmaxf(ylo - hiy, loy - (ylo + wy)), 0.f);
                    const float ddz = fmaxf(fmaxf(zlo - hiz, loz - (zlo + wz)), 0.f);
                    const float ch2 = reach2 - ddy * ddy - ddz * ddz;
                    if (ch2 > 0.f) {
                        const float ch = fmaf(ch2 * rsqrtf(ch2), 1.0001f, 1e-4f);
                        const int ca = max(ux0, (int)floorf((lox - ch) * A.inv_w.x));
                        const int cb = min(ux1, (int)floorf((hix + ch) * A.inv_w.x));
                        int ky = 0, kz = 0, cy = uy, cz = uz;
                        while (cy < 0) { cy += A.nc.y; --ky; }
                        while (cy >= A.nc.y) { cy -= A.nc.y; ++ky; }
                        while (cz < 0) { cz += A.nc.z; --kz; }
                        while (cz >= A.nc.z) { cz -= A.nc.z; ++kz; }
                        const int kx = kx0 + piece;
                        const int xa = max(ca, kx * A.nc.x) - kx * A.nc.x;
                        const int xb = min(cb, (kx + 1) * A.nc.x - 1) - kx * A.nc.x;
                        if (xa <= xb) {
                            const int rowbase = (cz * A.nc.y + cy) * A.nc.x;
                            beg = A.cell_start[rowbase + xa];
                            len = A.cell_start[rowbase + xb + 1] - beg;
                            sx = (float)kx * A.L.x;
                            sy = (float)ky * A.L.y;
                            sz = (float)kz * A.L.z;
                        }
                    }
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

            // candidates are loaded one round ahead of their culling, so that
            // the loads of round k+1 are in flight while round k is culled and
            // the chunk is tested
            int sc = 0;   // this lane's segment cursor
            float4 nq[TM_UNROLL];
            int ns[TM_UNROLL];
            auto load_round = [&](int t0) {
#pragma unroll
                for (int u = 0; u < TM_UNROLL; ++u) {
                    const int t = t0 + u * 32 + lane;
                    ns[u] = -1;
                    if (t < total) {
                        while (W.seg[sc + 1].pre <= t) ++sc;
                        ns[u] = sc;
                        nq[u] = A.pos_cell[W.seg[sc].beg + (t - W.seg[sc].pre)];
                    }
                }
            };
            load_round(0);
            for (int t0 = 0; t0 < total; t0 += 32 * TM_UNROLL) {
                float4 q[TM_UNROLL];
                int qs[TM_UNROLL];
#pragma unroll
                for (int u = 0; u < TM_UNROLL; ++u) {
                    q[u] = nq[u];
                    qs[u] = ns[u];
                }
                if (t0 + 32 * TM_UNROLL < total) load_round(t0 + 32 * TM_UNROLL);
                if (ncand > TM_CH - 32 * TM_UNROLL) test_chunk(false);
#pragma unroll
                for (int u = 0; u < TM_UNROLL; ++u) {
                    bool keep = false;
                    float4 c = q[u];
                    if (qs[u] >= 0) {
                        const SegEntry& e = W.seg[qs[u]];
                        c.x += e.sx;
                        c.y += e.sy;
                        c.z += e.sz;
                        const float ex = fmaxf(fmaxf(lox - c.x, c.x - hix), 0.f);
                        const float ey = fmaxf(fmaxf(loy - c.y, c.y - hiy), 0.f);
                        const float ez = fmaxf(fmaxf(loz - c.z, c.z - hiz), 0.f);
                        keep = fmaf(ez, ez, fmaf(ey, ey, ex * ex)) < reach2 &&
                               !(compact && (unsigned)(__float_as_int(c.w) - base) < 32u);
                    }
                    const unsigned bm = __ballot_sync(FULL, keep);
                    if (keep)
                        stage_cand(W, ncand + __popc(bm & lt_mask), c.x - ox, c.y - oy, c.z - oz,
                                   __float_as_int(c.w));
                    ncand += __popc(bm);
                }
            }
            __syncwarp();
        }
        test_chunk(true);

        // the rest of the buffer: a last group of TM_GROUP completed with pads
        // where the row has room for it (pad-filled rows), else one by one
        drain();
        int filled = done;                 // slots of the row written so far (from 0)
        if (VW >= 4 && A.pad_fill && pend > 0 && done + TM_GROUP <= cap) {
            int v[TM_GROUP];
#pragma unroll
            for (int e = 0; e < TM_GROUP; ++e) v[e] = e < pend ? buf[e * 32] : -1;
            if (VW == 8) {
                st_global_v8(row + done, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
            } else {
                st_global_v4(row + done, v[0], v[1], v[2], v[3]);
                st_global_v4(row + done + 4, v[4], v[5], v[6], v[7]);
            }
            filled = done + TM_GROUP;
        } else {
            for (int e = 0; e < pend; ++e)
                if (done + e < cap) row[done + e] = buf[e * 32];
            filled = min(done + pend, cap);
        }
        const int cnt = done + pend;
        if (!valid) filled = cap;

        if (valid) A.counts[i] = cnt;
        if (A.pad_fill && valid) {
            // each lane pads its own row (the kernel is bound by instruction
            // issue, not by the L1 pipe, so few wide stores beat a coalesced
            // pass over the 32 rows)
            int e = filled;
            if (VW == 8) {
                for (; e < cap && (e & 7); ++e) row[e] = -1;
                for (; e + 8 <= cap; e += 8) st_global_v8(row + e, -1, -1, -1, -1, -1, -1, -1, -1);
            } else if (VW == 4) {
                for (; e < cap && (e & 3); ++e) row[e] = -1;
                for (; e + 4 <= cap; e += 4) st_global_v4(row + e, -1, -1, -1, -1);
            }
            for (; e < cap; ++e) row[e] = -1;
        }
        const unsigned ov = __ballot_sync(FULL, valid && cnt > cap);
        if (ov && lane == 0) atomicOr(A.status, TESS_DEV_OVERFLOW);
        __syncwarp();
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
    if ((flags & ~(TESS_NO_PAD_FILL | TESS_LANE_SEARCH | TESS_TILE_SEARCH)) != 0) return TESS_ERR_INVALID_ARG;
    if ((flags & TESS_LANE_SEARCH) && (flags & TESS_TILE_SEARCH)) return TESS_ERR_INVALID_ARG;
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
        cell_scatter_kernel<<<blocks, 256, 0, s>>>(L.cell_id, L.cell_rank, n, L.cell_start, L.slot_atom, overflow);
        cell_order_kernel<<<(int)std::min<long long>((m + 255) / 256, (long long)sms * 16), 256, 0, s>>>(
            L.slot_atom, m, L.cell_start, pos4, L.pos_cell);
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
        const bool want_lane = (flags & TESS_LANE_SEARCH) || (!(flags & TESS_TILE_SEARCH) && TESS_DEFAULT_LANE);
        if (want_lane && lane_ok) {
            const long long blocks = (ntiles + PL_WARPS - 1) / PL_WARPS;
            pair_search_lane_kernel<<<(unsigned)std::min<long long>(blocks, 1LL << 30), PL_WARPS * 32, 0, s>>>(A);
        } else {
#if TESS_TM_RANGES
            const long long blocks = std::min<long long>((ntiles + TM_WARPS - 1) / TM_WARPS, (long long)sms * 4);
#else
            const long long blocks = std::min<long long>((ntiles + TM_WARPS - 1) / TM_WARPS, 1LL << 30);
#endif
            const bool v8 = cap % 8 == 0 && aligned(nbr, 32), v4 = cap % 4 == 0 && aligned(nbr, 16);
            auto launch = [&](auto kern) {
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TM_SMEM);
                kern<<<(unsigned)blocks, TM_WARPS * 32, TM_SMEM, s>>>(A);
            };
            if (v8) launch(pair_tile_kernel<8>);
            else if (v4) launch(pair_tile_kernel<4>);
            else launch(pair_tile_kernel<1>);
        }
        count_launch();
    }
    return launch_status();
}

}  // namespace tess
