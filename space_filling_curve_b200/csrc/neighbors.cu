// neighbors.cu -- fixed-capacity Verlet list at rs = rc + skin (shapes held
// constant between rebuilds, a neighbor search in three levels; Tessera,
// abstract).
//
// Level 0 (binning, deterministic):
//   cell_count     cell id per atom, histogram (one atomic per run of equal
//                  cells in a warp)
//   row_pad        (record layout) an odd cell row gets a pad slot
//   scan_*         exclusive scan of the cell counts -> cell_start
//   cell_scatter   atom indices into their cells (any order within a cell)
//   cell_order     within each cell, order by atom index and write the
//                  positions in cell order: as two-slot records (x0 x1 | y0 y1
//                  | z0 z1 | i0 i1) with every cell row starting at an even
//                  slot for the default search, as float4 (x, y, z, index
//                  bits) for the other two
// Levels 1-3, three kernels with the same lists (rows in different orders):
//   pair_search_duo_kernel (TESS_LANE2_SEARCH, the default): two atoms per
//     lane; each walks the 5 x 5 cell rows around its row, clipped to the
//     atoms' chords (level 1-2), and tests every record of the windows
//     against both atoms in packed f32x2 (level 3), accepted indices staged
//     per atom in shared memory and drained to the rows in 32-byte groups
//   pair_search_lane_kernel (TESS_LANE_SEARCH): the same walk with one atom
//     per lane over float4 candidates
//   pair_tile_kernel (TESS_TILE_SEARCH; boxes shorter than 2 reach): one warp
//     per 32 Hilbert-consecutive atoms; the cell rows within reach of their
//     bounding box, culled against it and compacted into a shared chunk,
//     tested by every lane (broadcast reads), 32 candidates per accept mask.
// Which one runs when the caller names none is TESS_DEFAULT_SEARCH.
#include <climits>
#include <type_traits>

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
// per-lane stencils rely on width >= rs/CELL_DIV along y and z, which
// coarsening keeps), xfine times narrower along x (the per-lane searches clip
// each cell row to a chord along x, so narrower x cells mean fewer
// candidates), coarsened when that would give more than ~2 cells per atom.
static Grid make_grid(int n, tess_box box, float rs, double xfine) {
    Grid g{};
    const float L[3] = {box.lx, box.ly, box.lz};
    double w = (double)rs * 1.0001 / (double)CELL_DIV;
    for (int it = 0; it < 64; ++it) {
        long long tot = 1;
        for (int d = 0; d < 3; ++d) {
            long long c = (long long)std::floor((double)L[d] / (d == 0 ? w / xfine : w));
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
    pdl_wait();
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
        // one atomic per run of lanes in the same cell; each lane keeps its
        // slot among the cell's atoms (any order: cell_order fixes it)
        const WarpRun g = warp_run((unsigned)c, valid);
        const int lane = threadIdx.x & 31;
        int b0 = 0;
        if (valid && lane == g.leader) b0 = atomicAdd(&cnt[c], g.len);
        b0 = __shfl_sync(FULL, b0, valid ? g.leader : lane);
        if (valid) cell_rank[i] = b0 + g.rank;
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0 && status) atomicOr(status, TESS_DEV_BAD_INPUT);
}

__global__ void cell_scatter_kernel(const int* __restrict__ cell_id, const int* __restrict__ cell_rank, int n,
                                    long long nslots, const int* __restrict__ cell_start,
                                    int* __restrict__ slot_atom, int32_t* status) {
    pdl_wait();
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const long long slot = (long long)cell_start[cell_id[i]] + cell_rank[i];
        if (check_index(slot, nslots, status)) slot_atom[slot] = i;
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

// Batcher's odd-even merge network for 8 keys (19 comparators).
__device__ __forceinline__ void sort8(int (&v)[8]) {
    cswap(v[0], v[1]); cswap(v[2], v[3]); cswap(v[4], v[5]); cswap(v[6], v[7]);
    cswap(v[0], v[2]); cswap(v[1], v[3]); cswap(v[4], v[6]); cswap(v[5], v[7]);
    cswap(v[1], v[2]); cswap(v[5], v[6]);
    cswap(v[0], v[4]); cswap(v[1], v[5]); cswap(v[2], v[6]); cswap(v[3], v[7]);
    cswap(v[2], v[4]); cswap(v[3], v[5]);
    cswap(v[1], v[2]); cswap(v[3], v[4]); cswap(v[5], v[6]);
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
            sort8(v);
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

// Two-slot records for the two-atoms-per-lane search: slots 2m and 2m + 1
// of the cell order in one 32-byte record, coordinates and indices paired so
// that one 256-bit load yields (x0 x1), (y0 y1), (z0 z1) as packed f32x2
// operands.  In this layout every cell row starts at an even slot: a row
// holding an odd number of atoms ends with one pad slot (index -1, NaN
// coordinates), which fails every distance test.
struct alignas(32) SlotPair {
    float x[2], y[2], z[2];
    int i[2];
};

// One warp per cell row: the row's atom count; an odd count gets its pad
// slot counted in the row's last cell, so the scan of the counts starts every
// row at an even slot.  rowpad[r] = 1 marks such a row.
__global__ void row_pad_kernel(int* __restrict__ cnt, int ncx, long long nrows, int* __restrict__ rowpad) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < nrows; r += warps) {
        const int* row = cnt + r * ncx;
        int sum = 0;
        for (int x = lane; x < ncx; x += 32) sum += row[x];
        sum = (int)__reduce_add_sync(FULL, (unsigned)sum);
        if (lane == 0) {
            rowpad[r] = sum & 1;
            if (sum & 1) cnt[r * ncx + ncx - 1] += 1;
        }
    }
}

__device__ __forceinline__ void put_slot(SlotPair* pairs, int s, float x, float y, float z, int i) {
    float* f = reinterpret_cast<float*>(pairs + (s >> 1)) + (s & 1);
    f[0] = x;
    f[2] = y;
    f[4] = z;
    reinterpret_cast<int*>(f)[6] = i;
}

// Both slots of record r in one 32-byte store (a plain store: the search
// reads the records next).
__device__ __forceinline__ void put_record(SlotPair* pairs, int r, float4 p0, int i0, float4 p1, int i1) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(pairs + r),
                 "r"(__float_as_int(p0.x)), "r"(__float_as_int(p1.x)), "r"(__float_as_int(p0.y)),
                 "r"(__float_as_int(p1.y)), "r"(__float_as_int(p0.z)), "r"(__float_as_int(p1.z)), "r"(i0), "r"(i1)
                 : "memory");
}

// cell_order for the record layout: the same order inside each cell, the
// positions written as two-slot records (a record whose two slots both
// belong to the cell, its pad slot included, in one store; a record shared
// with a neighboring cell half by half), and the pad slot of an odd row
// (the last slot of the row's last cell) filled.  One thread per cell; the
// range and the first two atom indices are loaded first (most cells hold at
// most two atoms), the others only for a larger cell.
struct CellLoad {
    int b, e, m;
    bool pad;
    int v0, v1;   // the cell's first two atom indices (most cells hold at most two)
};

__device__ __forceinline__ void cell_load(CellLoad& L, long long c, const int* __restrict__ slot_atom, int ncx,
                                          const int* __restrict__ cell_start, const int* __restrict__ rowpad) {
    L.b = cell_start[c];
    L.e = cell_start[c + 1];
    const long long r = c / ncx;
    L.pad = c - r * ncx == ncx - 1 && rowpad[r];
    if (L.pad) --L.e;                  // slot e is the row's pad
    L.m = L.e - L.b;
    L.v0 = L.m > 0 ? slot_atom[L.b] : INT_MAX;
    L.v1 = L.m > 1 ? slot_atom[L.b + 1] : INT_MAX;
}

__device__ __forceinline__ void cell_emit(const CellLoad& L, const int* __restrict__ slot_atom,
                                          const float4* __restrict__ pos, SlotPair* __restrict__ pairs) {
    const float nan = __int_as_float(0x7fc00000);
    const float4 pnan = make_float4(nan, nan, nan, nan);
    const int b = L.b, e = L.e, m = L.m;
    const bool pad = L.pad;
    if (m <= 0) {
        if (pad) put_slot(pairs, e, nan, nan, nan, -1);
        return;
    }
    if (m <= 8) {
        int v[8];
        v[0] = L.v0;
        v[1] = L.v1;
#pragma unroll
        for (int k = 2; k < 8; ++k) v[k] = k < m ? slot_atom[b + k] : INT_MAX;
        if (m <= 2) cswap(v[0], v[1]);
        else sort8(v);
        // slots b .. e-1 hold v[0 .. m-1], slot e the pad when there is one
        // (the pad is always the second half of its record)
        auto emit = [&](auto first) {
            constexpr int K0 = decltype(first)::value;
            if (K0 == 1) {             // slot b: the second half of a record shared with the cell before
                const float4 p = pos[v[0]];
                put_slot(pairs, b, p.x, p.y, p.z, v[0]);
            }
#pragma unroll
            for (int kk = K0; kk < 8; kk += 2) {
                if (kk + 1 < m) {
                    put_record(pairs, (b + kk) >> 1, pos[v[kk]], v[kk], pos[v[kk + 1]], v[kk + 1]);
                } else if (kk + 1 == m) {
                    const float4 p = pos[v[kk]];
                    if (pad) put_record(pairs, (b + kk) >> 1, p, v[kk], pnan, -1);
                    else put_slot(pairs, b + kk, p.x, p.y, p.z, v[kk]);   // shared with the cell after
                }
            }
        };
        if (b & 1) emit(std::integral_constant<int, 1>{});
        else emit(std::integral_constant<int, 0>{});
    } else {
        for (int s = b; s < e; ++s) {
            const int i = slot_atom[s];
            int rk = 0;
            for (int t = b; t < e; ++t) rk += slot_atom[t] < i;
            const float4 p = pos[i];
            put_slot(pairs, b + rk, p.x, p.y, p.z, i);
        }
        if (pad) put_slot(pairs, e, nan, nan, nan, -1);
    }
}

// 32 registers, so that 8 blocks of 256 threads fit an SM: the kernel waits
// on its chain of dependent loads (range, indices, positions), and more
// threads in flight beat holding two cells per thread.
__global__ __launch_bounds__(256, 8) void cell_order_pairs_kernel(const int* __restrict__ slot_atom, long long ncell,
                                                                 int ncx, const int* __restrict__ cell_start,
                                                                 const int* __restrict__ rowpad,
                                                                 const float4* __restrict__ pos,
                                                                 SlotPair* __restrict__ pairs) {
    pdl_wait();
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < ncell; c += stride) {
        CellLoad L;
        cell_load(L, c, slot_atom, ncx, cell_start, rowpad);
        cell_emit(L, slot_atom, pos, pairs);
    }
}

// ---------------------------------------------------------------- pair search

constexpr int PS_BUF = 32;           // per-lane staging of accepted indices, per-lane search
constexpr int PS_GROUP = 8;          // accepted indices leave in aligned groups of 8 (32 bytes)

struct SlotPair;

struct PairArgs {
    const float4* pos;
    const float4* pos_cell;
    const SlotPair* pairs;   // two-slot records (the two-atoms-per-lane search)
    const int* nslots;       // slots of the record layout, pads included (device)
    const int* cell_start;
    int n;
    int cap;
    int pad_fill;
    int vec_rows;      // rows can take 16-byte stores (cap % 4 == 0, 16-byte aligned nbr)
    int vec8;          // rows can take 32-byte stores (cap % 8 == 0, 32-byte aligned nbr)
    int row_tiles;     // tiles of 32 records per cell row, on average (at least 1)
    int far_cells;     // two atoms of one row more than this many cells apart take two passes
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

        // the complete groups of TM_GROUP buffered indices to the row, the
        // newest first: the remainder (the oldest) stays at the front of the
        // buffer (the order within a row is free)
        auto drain = [&]() {
            const int groups = pend / TM_GROUP;
            const int rest = pend - groups * TM_GROUP;
            for (int gi = 0; gi < groups; ++gi) {
                const int* src = buf + (rest + gi * TM_GROUP) * 32;
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
        // full groups to the row, the newest first: the remainder (the oldest)
        // stays at the front of the column (the order within a row is free)
        auto drain = [&](bool all) {
            const int pend = (int)((wsa - buf_sa) >> 7);
            const int groups = pend / PS_GROUP;
            const int rest = pend - groups * PS_GROUP;
            for (int gi = 0; gi < groups; ++gi) {
                const int* src = buf + (rest + gi * PS_GROUP) * 32;
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
            if (all) {
                for (int e = 0; e < rest; ++e)
                    if (done + e < cap) row[done + e] = buf[e * 32];
                done += rest;
                wsa = buf_sa;
            } else {
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

// ------------------------------------------------ two atoms per lane
//
// pair_search_duo_kernel (TESS_LANE2_SEARCH): the per-lane stencil walk with
// two atoms per lane, over the two-slot records.  A warp takes 32
// consecutive records (64 slots) of the cell order; lane l owns the atoms in
// slots 2l and 2l + 1 of them, which lie in one cell row (every row starts at
// an even slot).  For each of the 5 x 5 cell rows around that row the lane
// walks the union of its two atoms' x windows (each clipped to that atom's
// chord at the row's distance) record by record: one 32-byte load feeds four
// distance tests -- two candidates against two atoms -- in packed f32x2
// arithmetic.  Where the two windows together would span more than a row
// (two atoms far apart in a sparse row) the lane walks them one after the
// other instead.  Accepted indices are staged per atom in shared memory and
// leave for the atom's row in aligned 32-byte groups.

#ifndef TESS_PD_WARPS
#define TESS_PD_WARPS 4
#endif
#ifndef TESS_PD_BUF
#define TESS_PD_BUF 20
#endif
#ifndef TESS_PD_GROUP
#define TESS_PD_GROUP 1
#endif
constexpr int PD_WARPS = TESS_PD_WARPS;
constexpr int PD_BUF = TESS_PD_BUF;        // staged indices per atom (two buffers per lane)
#ifndef TESS_PD_CHUNK
#define TESS_PD_CHUNK 2
#endif
constexpr int PD_CHUNK = TESS_PD_CHUNK;    // records per lane between buffer votes

typedef unsigned long long u64;

// The record at a (32-byte aligned) into four packed pairs when p; the
// registers keep their values otherwise.
__device__ __forceinline__ void ld_pair_if(bool p, const SlotPair* a, u64& x, u64& y, u64& z, u64& j) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
        "@p ld.global.nc.v4.b64 {%0, %1, %2, %3}, [%4];\n\t}"
        : "+l"(x), "+l"(y), "+l"(z), "+l"(j)
        : "l"(a), "r"((int)p));
}

// Four tests of one record (slots k, k + 1) against atoms a and b: element 0
// counts when beg <= k < end, element 1 when k + 1 < end; with SELF the
// lane's own record (k == own) skips a against itself (element 0) and b
// against itself (element 1).  Each accepted index is appended to its atom's
// staging column (wa, wb: shared addresses, 128-byte steps).
// Four tests of one record against atoms a and b (packed pairs qa*, qb*),
// counted when `live`; with SELF the lane's own record (k == own) skips a
// against itself (element 0) and b against itself (element 1).  Each accepted
// index is appended to its atom's staging column (wa, wb: shared addresses,
// 128-byte steps; the store happens either way and a rejected index is
// overwritten by the next).
#define TESS_DUO_BODY(SA, SB)                                \
    "{\n\t.reg .b64 dx, dy, dz, r;\n\t.reg .f32 r0, r1;\n\t"  \
    ".reg .b32 j0, j1;\n\t.reg .pred v, sa, sb, p;\n\t"      \
    "setp.ne.b32 v, %13, 0;\n\t"                              \
    SA SB                                                     \
    "mov.b64 {j0, j1}, %5;\n\t"                               \
    "sub.rn.f32x2 dx, %2, %6;\n\t"                            \
    "sub.rn.f32x2 dy, %3, %7;\n\t"                            \
    "sub.rn.f32x2 dz, %4, %8;\n\t"                            \
    "mul.rn.f32x2 r, dx, dx;\n\t"                             \
    "fma.rn.f32x2 r, dy, dy, r;\n\t"                          \
    "fma.rn.f32x2 r, dz, dz, r;\n\t"                          \
    "mov.b64 {r0, r1}, r;\n\t"                                \
    "setp.lt.and.f32 p, r0, %12, sa;\n\t"                     \
    "st.shared.b32 [%0], j0;\n\t"                             \
    "@p add.u32 %0, %0, 128;\n\t"                             \
    "setp.lt.and.f32 p, r1, %12, v;\n\t"                      \
    "st.shared.b32 [%0], j1;\n\t"                             \
    "@p add.u32 %0, %0, 128;\n\t"                             \
    "sub.rn.f32x2 dx, %2, %9;\n\t"                            \
    "sub.rn.f32x2 dy, %3, %10;\n\t"                           \
    "sub.rn.f32x2 dz, %4, %11;\n\t"                           \
    "mul.rn.f32x2 r, dx, dx;\n\t"                             \
    "fma.rn.f32x2 r, dy, dy, r;\n\t"                          \
    "fma.rn.f32x2 r, dz, dz, r;\n\t"                          \
    "mov.b64 {r0, r1}, r;\n\t"                                \
    "setp.lt.and.f32 p, r0, %12, v;\n\t"                      \
    "st.shared.b32 [%1], j0;\n\t"                             \
    "@p add.u32 %1, %1, 128;\n\t"                             \
    "setp.lt.and.f32 p, r1, %12, sb;\n\t"                     \
    "st.shared.b32 [%1], j1;\n\t"                             \
    "@p add.u32 %1, %1, 128;\n\t}"

template <bool SELF>
__device__ __forceinline__ void duo_test(unsigned& wa, unsigned& wb, u64 x, u64 y, u64 z, u64 j, u64 qax,
                                         u64 qay, u64 qaz, u64 qbx, u64 qby, u64 qbz, float rs2, bool live, int k,
                                         int own) {
    if (SELF) {
        asm volatile(TESS_DUO_BODY("setp.ne.and.s32 sa, %14, %15, v;\n\t", "setp.ne.and.s32 sb, %14, %15, v;\n\t")
                     : "+r"(wa), "+r"(wb)
                     : "l"(x), "l"(y), "l"(z), "l"(j), "l"(qax), "l"(qay), "l"(qaz), "l"(qbx), "l"(qby), "l"(qbz),
                       "f"(rs2), "r"((int)live), "r"(k), "r"(own)
                     : "memory");
    } else {
        asm volatile(TESS_DUO_BODY("mov.pred sa, v;\n\t", "mov.pred sb, v;\n\t")
                     : "+r"(wa), "+r"(wb)
                     : "l"(x), "l"(y), "l"(z), "l"(j), "l"(qax), "l"(qay), "l"(qaz), "l"(qbx), "l"(qby), "l"(qbz),
                       "f"(rs2), "r"((int)live), "r"(k), "r"(own)
                     : "memory");
    }
}
#undef TESS_DUO_BODY

#ifndef TESS_PD_BULKPAD
#define TESS_PD_BULKPAD 1
#endif
constexpr int PD_PADS = 256;               // ints of -1 that the pad copies read

// bytes (a multiple of 16) from shared address src to global dst (both 16-byte
// aligned) by the bulk copy engine, as one bulk group of this thread
__device__ __forceinline__ void bulk_store(int* dst, unsigned src, unsigned bytes) {
    asm volatile(
        "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n\t"
        "cp.async.bulk.commit_group;" ::"l"(dst), "r"(src), "r"(bytes)
        : "memory");
}

#ifndef TESS_PD_MINB
#define TESS_PD_MINB 7
#endif

__global__ __launch_bounds__(PD_WARPS * 32, TESS_PD_MINB) void pair_search_duo_kernel(PairArgs A) {
    pdl_wait();
    __shared__ int s_buf[PD_WARPS][2][32 * PD_BUF];
#if TESS_PD_BULKPAD
    __shared__ __align__(16) int s_pads[PD_PADS];
    for (int k = threadIdx.x; k < PD_PADS; k += blockDim.x) s_pads[k] = -1;
    // the bulk copies read s_pads through the async proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    const unsigned pads_sa = (unsigned)__cvta_generic_to_shared(s_pads);
#endif
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int* const bufa = &s_buf[warp][0][lane];
    int* const bufb = &s_buf[warp][1][lane];
    const unsigned basea = (unsigned)__cvta_generic_to_shared(bufa);
    const unsigned baseb = (unsigned)__cvta_generic_to_shared(bufb);
    const int cap = A.cap, ncx = A.nc.x;
    const int nrec = *A.nslots >> 1;
    const long long ntiles = ((long long)nrec + 31) / 32;
    const float wy = (float)A.L.y / (float)A.nc.y, wz = (float)A.L.z / (float)A.nc.z;
    const float reach2 = A.reach * A.reach;
    const float nan = __int_as_float(0x7fc00000);
    const unsigned vote_at = (unsigned)(PD_BUF - 2 * PD_CHUNK) * 128u;

    // full groups of 8 staged indices to the row: the newest ones, so that
    // the remainder (the oldest, fewer than 8) stays at the front of the
    // column and nothing moves (the order within a row is free)
    auto drain = [&](int* buf, unsigned base, unsigned& w, int& done, int* row) {
        const int pend = (int)((w - base) >> 7);
        const int groups = pend >> 3;
        const int rest = pend - groups * 8;
        for (int g = 0; g < groups; ++g) {
            const int* src = buf + (rest + g * 8) * 32;
            if (A.vec8 && done + 8 <= cap) {
                st_global_v8(row + done, src[0], src[32], src[64], src[96], src[128], src[160], src[192], src[224]);
            } else {
                for (int e = 0; e < 8; ++e)
                    if (done + e < cap) row[done + e] = src[e * 32];
            }
            done += 8;
        }
        w = base + 128u * (unsigned)rest;
    };
    // the last staged indices (a group completed with pads where the row is
    // pad-filled and has room), the count, and the pads
    auto finish = [&](int* buf, unsigned base, unsigned w, int done, int* row, bool valid, int idx) {
        drain(buf, base, w, done, row);
        const int pend = (int)((w - base) >> 7);
        int filled;
        if (A.pad_fill && A.vec8 && pend > 0 && done + 8 <= cap) {
            int v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = e < pend ? buf[e * 32] : -1;
            st_global_v8(row + done, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
            filled = done + 8;
        } else {
            for (int e = 0; e < pend; ++e)
                if (done + e < cap) row[done + e] = buf[e * 32];
            filled = min(done + pend, cap);
        }
        const int cnt = done + pend;
        if (valid) {
            A.counts[idx] = cnt;
            if (A.pad_fill) {
                int e = filled;
                if (A.vec8) {
                    for (; e < cap && (e & 7); ++e) row[e] = -1;
#if TESS_PD_BULKPAD
                    // the pads as bulk copies of a shared block of -1 (the copy
                    // engine writes them, not the lane's load/store path)
                    while (e + 8 <= cap) {
                        const int m8 = min((cap - e) >> 3, PD_PADS >> 3);
                        bulk_store(row + e, pads_sa, (unsigned)m8 * 32u);
                        e += m8 * 8;
                    }
#else
                    for (; e + 8 <= cap; e += 8) st_global_v8(row + e, -1, -1, -1, -1, -1, -1, -1, -1);
#endif
                }
                for (; e < cap; ++e) row[e] = -1;
            }
        }
        return cnt;
    };

    u64 cx[PD_CHUNK], cy2[PD_CHUNK], cz2[PD_CHUNK], cj[PD_CHUNK];
#pragma unroll
    for (int u = 0; u < PD_CHUNK; ++u) cx[u] = cy2[u] = cz2[u] = cj[u] = 0ull;

    for (long long pos = (long long)blockIdx.x * PD_WARPS + warp; pos < ntiles;
         pos += (long long)gridDim.x * PD_WARPS) {
        // the warps of a block take tiles about one cell row apart (row_tiles
        // tiles per row on average): the same x range of adjacent rows, whose
        // stencils share most of their cell rows in L1
        long long tile = pos;
        if (TESS_PD_GROUP) {
            const long long span = (long long)PD_WARPS * A.row_tiles, g = pos / span;
            if ((g + 1) * span <= ntiles) {
                const long long r = pos - g * span;
                tile = g * span + (r % PD_WARPS) * A.row_tiles + r / PD_WARPS;
            }
        }
        const int m = (int)(tile * 32) + lane;
        u64 ox = 0ull, oy = 0ull, oz = 0ull, oj = ~0ull;
        ld_pair_if(m < nrec, A.pairs + m, ox, oy, oz, oj);
        const int ia = (int)(unsigned)oj, ib = (int)(oj >> 32);
        const bool va = ia >= 0, vb = ib >= 0;
        // test coordinates as given (NaN for a pad); the windows use them too,
        // with x clamped into the box (y and z only enter through distances
        // to cell rows, where a NaN or distant value just empties the row)
        const float3 pa = make_float3(__uint_as_float((unsigned)ox), __uint_as_float((unsigned)oy),
                                      __uint_as_float((unsigned)oz));
        const float3 pb = make_float3(__uint_as_float((unsigned)(ox >> 32)), __uint_as_float((unsigned)(oy >> 32)),
                                      __uint_as_float((unsigned)(oz >> 32)));
        const float xa = fminf(fmaxf(pa.x, 0.f), A.L.x), xb = fminf(fmaxf(pb.x, 0.f), A.L.x);
        int* const rowa = A.nbr + (size_t)(va ? ia : 0) * cap;
        int* const rowb = A.nbr + (size_t)(vb ? ib : 0) * cap;
        const int cyc = cell_coord(pa.y, A.inv_w.y, A.nc.y);
        const int czc = cell_coord(pa.z, A.inv_w.z, A.nc.z);
        const int own = 2 * m;
        // two atoms whose windows together could exceed nc.x + 1 cells (far
        // apart in a sparse row) are walked one after the other, b in a
        // second pass
        const bool far = vb && cell_coord(xb, A.inv_w.x, ncx) - cell_coord(xa, A.inv_w.x, ncx) > A.far_cells;
        const int passes = __any_sync(FULL, far) ? 2 : 1;

        int donea = 0, doneb = 0;
        unsigned wa = basea, wb = baseb;

        for (int pass = 0; pass < passes; ++pass) {
            const bool usea = va && pass == 0, useb = vb && (pass == 0) != far;
            for (int dz = -CELL_DIV; dz <= CELL_DIV; ++dz) {
                int wz_i = czc + dz, kz = 0;
                while (wz_i < 0) { wz_i += A.nc.z; --kz; }
                while (wz_i >= A.nc.z) { wz_i -= A.nc.z; ++kz; }
                const float zlo = (float)(czc + dz) * wz;
                const float dza = fmaxf(fmaxf(zlo - pa.z, pa.z - (zlo + wz)), 0.f);
                const float dzb = fmaxf(fmaxf(zlo - pb.z, pb.z - (zlo + wz)), 0.f);
                const u64 qaz = pk2(pa.z - (float)kz * A.L.z), qbz = pk2(pb.z - (float)kz * A.L.z);
                for (int dy = -CELL_DIV; dy <= CELL_DIV; ++dy) {
                    int wy_i = cyc + dy, ky = 0;
                    while (wy_i < 0) { wy_i += A.nc.y; --ky; }
                    while (wy_i >= A.nc.y) { wy_i -= A.nc.y; ++ky; }
                    const float ylo = (float)(cyc + dy) * wy;
                    const float dya = fmaxf(fmaxf(ylo - pa.y, pa.y - (ylo + wy)), 0.f);
                    const float dyb = fmaxf(fmaxf(ylo - pb.y, pb.y - (ylo + wy)), 0.f);
                    const float ch2a = reach2 - dya * dya - dza * dza;
                    const float ch2b = reach2 - dyb * dyb - dzb * dzb;
                    const u64 qay = pk2(pa.y - (float)ky * A.L.y), qby = pk2(pb.y - (float)ky * A.L.y);
                    const bool ina = usea && ch2a > 0.f, inb = useb && ch2b > 0.f;
                    // the union of the two x windows, in unwrapped cells
                    // (chords approximate, widened)
                    int lo = INT_MAX, hi = INT_MIN;
                    if (ina) {
                        const float ch = fmaf(ch2a * rsqrtf(ch2a), 1.0001f, 1e-4f);
                        lo = (int)floorf((xa - ch) * A.inv_w.x);
                        hi = (int)floorf((xa + ch) * A.inv_w.x);
                    }
                    if (inb) {
                        const float ch = fmaf(ch2b * rsqrtf(ch2b), 1.0001f, 1e-4f);
                        lo = min(lo, (int)floorf((xb - ch) * A.inv_w.x));
                        hi = max(hi, (int)floorf((xb + ch) * A.inv_w.x));
                    }
                    // as up to two ranges of slots; the second (wrapped) one
                    // has image shift kx + 1.  Slots just outside a range (a
                    // record's other half) lie in the same cell row beyond the
                    // window, so the distance test rejects them.
                    int B0 = 0, E0 = 0, B1 = 0, E1 = 0, k0 = 0, k1 = 0;
                    if (ina || inb) {
                        const int rowbase = (wz_i * A.nc.y + wy_i) * ncx;
                        int kx = 0;
                        while (lo < 0) { lo += ncx; hi += ncx; --kx; }
                        while (lo >= ncx) { lo -= ncx; hi -= ncx; ++kx; }
                        B0 = A.cell_start[rowbase + lo];
                        E0 = A.cell_start[rowbase + min(hi, ncx - 1) + 1];
                        k0 = kx;
                        if (hi >= ncx) {
                            B1 = A.cell_start[rowbase];
                            E1 = A.cell_start[rowbase + min(hi - ncx, ncx - 1) + 1];
                            k1 = kx + 1;
                            if (kx < 0) {
                                // the second range (image shift 0) holds the
                                // atoms' own cells: walk it first, in step with
                                // the main ranges of the other lanes
                                int t = B0; B0 = B1; B1 = t;
                                t = E0; E0 = E1; E1 = t;
                                k0 = kx + 1;
                                k1 = kx;
                            }
                        }
                    }

                    auto run = [&](auto self_tag) {
                        constexpr bool SELF = decltype(self_tag)::value;
#pragma unroll
                        for (int pc = 0; pc < 2; ++pc) {
                            const int beg = pc ? B1 : B0, end = pc ? E1 : E0;
                            const int kb = beg & ~1;
                            const int np = end > beg ? (end - kb + 1) >> 1 : 0;
                            const int maxp = (int)__reduce_max_sync(FULL, (unsigned)np);
                            if (maxp == 0) continue;
                            const float sx = (float)(pc ? k1 : k0) * A.L.x;
                            const u64 qax = pk2(usea ? pa.x - sx : nan), qbx = pk2(useb ? pb.x - sx : nan);
                            const SlotPair* src = A.pairs + (kb >> 1);
                            for (int t0 = 0; t0 < maxp; t0 += PD_CHUNK) {
                                if (__any_sync(FULL, max(wa - basea, wb - baseb) > vote_at)) {
                                    drain(bufa, basea, wa, donea, rowa);
                                    drain(bufb, baseb, wb, doneb, rowb);
                                }
#pragma unroll
                                for (int u = 0; u < PD_CHUNK; ++u)
                                    ld_pair_if(t0 + u < np, src + t0 + u, cx[u], cy2[u], cz2[u], cj[u]);
#pragma unroll
                                for (int u = 0; u < PD_CHUNK; ++u)
                                    duo_test<SELF>(wa, wb, cx[u], cy2[u], cz2[u], cj[u], qax, qay, qaz, qbx, qby,
                                                   qbz, A.rs2, t0 + u < np, kb + 2 * (t0 + u), own);
                            }
                        }
                    };
                    if (dz == 0 && dy == 0) run(std::true_type{});
                    else run(std::false_type{});
                }
            }
        }
        const int cnta = finish(bufa, basea, wa, donea, rowa, va, ia);
        const int cntb = finish(bufb, baseb, wb, doneb, rowb, vb, ib);
        const unsigned ov = __ballot_sync(FULL, (va && cnta > cap) || (vb && cntb > cap));
        if (ov && lane == 0) atomicOr(A.status, TESS_DEV_OVERFLOW);
        __syncwarp();
    }
#if TESS_PD_BULKPAD
    // s_pads must outlive the reads of this thread's bulk copies
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
#endif
}

// ---------------------------------------------------------------- host

struct NbrLayout {
    int* cell_id;
    int* cell_rank;
    int* cnt;
    unsigned long long* scan_state;   // look-back words of the offset scan
    size_t zero_words;                // cnt .. end of scan_state, zeroed per call
    int* cell_start;
    int* slot_atom;
    int* rowpad;
    float4* pos_cell;      // cell order as float4, or (same storage) as two-slot records
    SlotPair* pairs;
    int32_t* status;
    size_t total;
};

static NbrLayout nbr_layout(void* ws, int n, const Grid& g) {
    Carve c(ws);
    NbrLayout L{};
    const long long m = g.ncell;
    const long long nrows = (long long)g.nc[1] * g.nc[2];
    const long long slots = (long long)n + nrows;          // the record layout's pads included
    L.cell_id = c.take<int>((size_t)n);
    L.cell_rank = c.take<int>((size_t)n);
    L.cnt = c.take<int>((size_t)m);
    L.scan_state = c.take<unsigned long long>((size_t)scan_state_len(m));   // zeroed with cnt
    L.zero_words = (size_t)(reinterpret_cast<char*>(L.scan_state + scan_state_len(m)) -
                            reinterpret_cast<char*>(L.cnt)) / 4;
    L.cell_start = c.take<int>((size_t)m + 1);
    L.slot_atom = c.take<int>((size_t)slots);
    L.rowpad = c.take<int>((size_t)nrows);
    L.pairs = c.take<SlotPair>((size_t)((slots + 1) / 2));
    L.pos_cell = reinterpret_cast<float4*>(L.pairs);
    L.status = c.take<int32_t>(1);
    L.total = align_up(c.off, 256);
    return L;
}

static bool box_ok(tess_box b) { return finite_pos(b.lx) && finite_pos(b.ly) && finite_pos(b.lz); }

// x cells per y/z cell width for the two-atoms-per-lane search
#ifndef TESS_DUO_XFINE
#define TESS_DUO_XFINE 2.5
#endif

size_t build_neighbors_workspace(int n, tess_box box, float rc, float skin) {
    if (n <= 0 || !box_ok(box) || !(rc > 0.f) || !(skin >= 0.f)) return 0;
    const float rs = rc + skin;
    // enough for either grid (the search kind is chosen per call)
    return std::max(nbr_layout(nullptr, n, make_grid(n, box, rs, 1.0)).total,
                    nbr_layout(nullptr, n, make_grid(n, box, rs, TESS_DUO_XFINE)).total);
}

tess_status build_neighbors(const float* pos, int n, tess_box box, float rc, float skin, int cap, int flags,
                            void* ws, size_t ws_bytes, int32_t* nbr, int32_t* counts, int32_t* overflow,
                            cudaStream_t s) {
    if (n <= 0 || !pos || !ws || !nbr || !counts || !overflow || cap < 1) return TESS_ERR_INVALID_ARG;
    if (!box_ok(box) || !(rc > 0.f) || !(skin >= 0.f) || !std::isfinite(rc) || !std::isfinite(skin))
        return TESS_ERR_INVALID_ARG;
    const int kinds = flags & (TESS_LANE_SEARCH | TESS_TILE_SEARCH | TESS_LANE2_SEARCH);
    if ((flags & ~(TESS_NO_PAD_FILL | kinds)) != 0 || (kinds & (kinds - 1)) != 0) return TESS_ERR_INVALID_ARG;
    if (!aligned(pos, 16) || !aligned(ws, 256) || !aligned(nbr, 4) || !aligned(counts, 4)) return TESS_ERR_INVALID_ARG;
    const float rs = rc + skin;
    if (box.lx < 2.f * rs || box.ly < 2.f * rs || box.lz < 2.f * rs) return TESS_ERR_BOX_TOO_SMALL;
    // which search: the per-lane kinds need every box length >= 2 reach (a
    // window then wraps at most once); otherwise the tile search runs
    const float lmax = std::max(box.lx, std::max(box.ly, box.lz));
    const float reach = rs + 1e-3f + 4e-6f * lmax;
    const bool lane_ok = box.lx >= 2.f * reach && box.ly >= 2.f * reach && box.lz >= 2.f * reach;
    int kind = kinds ? kinds : TESS_DEFAULT_SEARCH;
    if (kind != TESS_TILE_SEARCH && !lane_ok) kind = TESS_TILE_SEARCH;
    const bool records = kind == TESS_LANE2_SEARCH;

    const Grid g = make_grid(n, box, rs, records ? TESS_DUO_XFINE : 1.0);
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

    {
        StageScope sc(ST_CELLS, s);
        zero2(reinterpret_cast<unsigned*>(overflow), 1, reinterpret_cast<unsigned*>(L.cnt), L.zero_words, sms, s);
        const int blocks = (int)std::min<long long>(((long long)n + 255) / 256, (long long)sms * 16);
        launch_pdl(cell_count_kernel, dim3(blocks), dim3(256), 0, s, (const float4*)pos4, n, nc, inv_w, Lb, L.cell_id,
                   L.cell_rank, L.cnt, overflow);
        const long long nrows = (long long)nc.y * nc.z;
        if (records) {
            const long long rb = std::min<long long>((nrows + 7) / 8, (long long)sms * 32);
            launch_pdl(row_pad_kernel, dim3((unsigned)rb), dim3(256), 0, s, L.cnt, nc.x, nrows, L.rowpad);
        }
        exclusive_scan(L.cnt, m, L.scan_state, L.cell_start, overflow, sms, s);
        launch_pdl(cell_scatter_kernel, dim3(blocks), dim3(256), 0, s, (const int*)L.cell_id, (const int*)L.cell_rank,
                   n, (long long)n + nrows, (const int*)L.cell_start, L.slot_atom, overflow);
        const int oblocks = (int)std::min<long long>((m + 255) / 256, (long long)sms * 16);
        if (records)
            launch_pdl(cell_order_pairs_kernel, dim3(oblocks), dim3(256), 0, s, (const int*)L.slot_atom, m, nc.x,
                       (const int*)L.cell_start, (const int*)L.rowpad, pos4, L.pairs);
        else
            cell_order_kernel<<<oblocks, 256, 0, s>>>(L.slot_atom, m, L.cell_start, pos4, L.pos_cell);
        count_launch(records ? 4 : 3);   // count, row pads, scatter, ordering (zero2 and the scan count themselves)
    }
    {
        StageScope sc(ST_PAIRS, s);
        PairArgs A;
        A.pos = pos4;
        A.pos_cell = L.pos_cell;
        A.pairs = L.pairs;
        A.nslots = L.cell_start + m;
        A.cell_start = L.cell_start;
        A.n = n;
        A.cap = cap;
        A.pad_fill = (flags & TESS_NO_PAD_FILL) ? 0 : 1;
        A.vec_rows = (cap % 4 == 0 && aligned(nbr, 16)) ? 1 : 0;
        A.vec8 = (cap % 8 == 0 && aligned(nbr, 32)) ? 1 : 0;
        A.row_tiles = 1;
        A.far_cells = 0;
        A.nc = nc;
        A.inv_w = inv_w;
        A.L = Lb;
        A.rs2 = rs * rs;
        A.reach = reach;
        A.nbr = nbr;
        A.counts = counts;
        A.status = overflow;
        const long long ntiles = ((long long)n + 31) / 32;
        if (kind == TESS_LANE2_SEARCH) {
            const long long recs = ((long long)n + (long long)nc.y * nc.z + 1) / 2;
            A.row_tiles = (int)std::max<long long>(1, std::llround((double)n / ((double)nc.y * nc.z) / 64.0));
            // a window reaches at most R cells either side of its atom's cell
            const double chmax = (double)reach * 1.0001 + 1e-4;
            A.far_cells = nc.x - 2 * ((int)std::ceil(chmax * (double)inv_w.x) + 1);
            const long long blocks = ((recs + 31) / 32 + PD_WARPS - 1) / PD_WARPS;
            launch_pdl(pair_search_duo_kernel, dim3((unsigned)std::min<long long>(blocks, 1LL << 30)),
                       dim3(PD_WARPS * 32), 0, s, A);
        } else if (kind == TESS_LANE_SEARCH) {
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
