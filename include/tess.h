/*
 * tess.h -- C ABI of the B200 neighbor-rebuild library (libtess.so).
 *
 * The library implements the per-rebuild neighbor pipeline of an
 * equivariant message-passing molecular-dynamics runtime, as described in
 * "Ab Initio Accuracy Beyond the Cutoff: Distributed Message-Passing
 * Equivariant Attention at Tens-of-Millions-of-Atom Scale" (Tessera),
 * abstract:
 *   - atoms are sorted along a space-filling curve (here the 3-D Hilbert
 *     curve)                                          -> tess_hilbert_sort
 *   - a neighbor list with fixed shapes between rebuilds, found by a
 *     three-level search (tile, cell, pair)           -> tess_build_neighbors
 *   - a conservative neighbor skin decides when to rebuild -> tess_skin_check
 *   - each message-passing layer aggregates one-hop neighbor features
 *     within the cutoff (review of arXiv 2505.06711, "load-bearing
 *     attack" paragraph)                              -> tess_edge_aggregate
 *
 * Conventions (all entry points):
 *   - Array pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing; scratch memory is a caller-provided workspace whose
 *     size the *_workspace query returns.  Workspaces must be 256-byte
 *     aligned; float4-layout arrays ([n,4] float) must be 16-byte aligned.
 *   - Every call is asynchronous on the given stream and does no host
 *     synchronisation.  The return value reports argument errors and launch
 *     errors (cudaGetLastError) only; conditions found on the device are
 *     written to caller-provided int32 words.
 *   - The periodic box is orthorhombic with its origin at 0; positions are
 *     expected in [0, L) per axis.
 *   - Indices are int32: n <= 2^31 - 1.  n_max for a workspace is the n the
 *     workspace was sized for.
 */
#ifndef TESS_H
#define TESS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* tess_stream_t;

typedef enum {
    TESS_OK = 0,
    TESS_ERR_INVALID_ARG = 1,        /* n <= 0, null pointer, bad parameter, misalignment */
    TESS_ERR_BOX_TOO_SMALL = 2,      /* some box length below 2 (rc + skin) */
    TESS_ERR_WORKSPACE_TOO_SMALL = 3,/* ws_bytes below the workspace query */
    TESS_ERR_CUDA = 4,               /* a kernel launch failed */
    TESS_ERR_TOO_LARGE = 5           /* n above the capacity of tess_hilbert_sort_static */
} tess_status;

/* Orthorhombic periodic box lengths (Angstrom, or any unit used throughout). */
typedef struct {
    float lx, ly, lz;
} tess_box;

/* Bits of the device status words (overflow / dev_status arguments). */
#define TESS_DEV_OVERFLOW   1   /* some neighbor count exceeded max_neighbors */
#define TESS_DEV_BAD_INPUT  2   /* some position outside [0, L) or not finite (clamped into the grid) */
#define TESS_DEV_TIMEOUT    4   /* an inter-block wait gave up; outputs of that call are invalid */
#define TESS_DEV_FULL_SORT  8   /* tess_hilbert_resort ran the full sort (its fast path did not apply) */
#define TESS_DEV_CHECK     16   /* checked builds (-DTESS_CHECK) only: a kernel met an index out of range
                                   and skipped that access */

/* tess_build_neighbors flags */
#define TESS_NO_PAD_FILL    1   /* leave slots >= min(count, max_neighbors) unwritten */
#define TESS_LANE_SEARCH    2   /* use the per-lane stencil search */
#define TESS_TILE_SEARCH    4   /* use the warp tile search (accept per 32-candidate block) */
#define TESS_LANE2_SEARCH   8   /* use the per-lane stencil search with two atoms per lane */

/* Human-readable name of a status code (static string). */
const char* tess_status_string(tess_status s);

/* Library version string (static). */
const char* tess_version(void);

/* Number of kernels this process has launched through the library so far (a
 * diagnostic counter; thread-safe). */
long long tess_kernel_launch_count(void);

/* ---------------------------------------------------------------------------
 * Hilbert sort -- Tessera orders the atoms along a space-filling curve
 * before cutting them into shards (Tessera, abstract).
 *
 * Each coordinate is quantised on a grid of 2^bits cells per axis: the scale
 * s = 2^bits / L is one fp32 division, the cell is floor(x * s) with x * s a
 * single fp32 multiply, clamped into [0, 2^bits - 1] (values below 0 or NaN
 * give 0).  The key is the 3-D Hilbert index of the cell (Skilling's
 * transform, "Programming the Hilbert curve", 2004; x is axis 0), 3*bits bits.
 * Atoms are ordered by key, ties by ascending input index, so the result is
 * unique.
 *
 *   pos          [n,3] float, input order (12-byte rows)
 *   bits         1..10 (10: a 1024^3 grid)
 *   ws, ws_bytes scratch of at least tess_hilbert_sort_workspace(n) bytes
 *   perm         [n] int32 out: perm[k] = input index of the atom at rank k
 *   keys_sorted  [n] uint32 out, nullable: key of the atom at rank k
 *   pos_sorted   [n,4] float out, nullable: (x, y, z, 0) of the atom at rank k
 *   dev_status   [1] int32 out, nullable: 0, or TESS_DEV_* bits
 *                (BAD_INPUT, TIMEOUT)
 * Errors: INVALID_ARG (n <= 0, null pos/perm/ws, bits outside 1..10, a
 * non-positive or non-finite box length, misaligned pos_sorted),
 * WORKSPACE_TOO_SMALL, CUDA.
 * ------------------------------------------------------------------------- */
size_t tess_hilbert_sort_workspace(int n);
tess_status tess_hilbert_sort(const float* pos, int n, tess_box box, int bits,
                              void* ws, size_t ws_bytes,
                              int32_t* perm, uint32_t* keys_sorted, float* pos_sorted,
                              int32_t* dev_status, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Incremental Hilbert re-sort -- the re-sort at a rebuild, after the atoms
 * have moved a little since the previous sort (Tessera re-sorts along its
 * curve at every rebuild; Tessera, abstract).
 *
 * Output: exactly what tess_hilbert_sort(pos, n, box, bits, ...) writes for
 * the same positions (perm, keys_sorted, pos_sorted, dev_status bits), for
 * any perm_prev / keys_prev.  It runs faster when they are the perm and
 * keys_sorted of an earlier sort of the same n atoms whose positions moved
 * little since: the call then starts from that order, fixes the atoms whose
 * key stayed within their old neighbors' keys with local block sorts, radix
 * sorts the few others and merges the two.  Its checks run on the device;
 * when one fails (perm_prev not a permutation, more than n/8 + 1024 atoms
 * far from their old place, a local run out of order) the call runs the full
 * sort instead and sets TESS_DEV_FULL_SORT in *dev_status.  No host
 * synchronisation either way.
 *
 *   pos        [n, 3] float, device, CURRENT positions in the original
 *              (unsorted) index order -- the same input as tess_hilbert_sort
 *   perm_prev  [n] int32, device: the earlier sort's perm
 *   keys_prev  [n] uint32, device: the earlier sort's keys_sorted
 *   perm, keys_sorted, pos_sorted, dev_status: as tess_hilbert_sort; they
 *              must not overlap perm_prev / keys_prev
 *   ws         tess_hilbert_resort_workspace(n) bytes, 256-byte aligned
 *              (about 19 n bytes plus small tables)
 * Errors: as tess_hilbert_sort, plus INVALID_ARG if perm_prev or keys_prev
 * is NULL.
 * ------------------------------------------------------------------------- */
size_t tess_hilbert_resort_workspace(int n);
tess_status tess_hilbert_resort(const float* pos, int n, tess_box box, int bits, const int32_t* perm_prev,
                                const uint32_t* keys_prev, void* ws, size_t ws_bytes, int32_t* perm,
                                uint32_t* keys_sorted, float* pos_sorted, int32_t* dev_status,
                                tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Morton (Z-order) sort -- the curve the Tessera abstract compares against:
 * it reports neighbor-search cost growing 1.7x along its curve and 3.0x
 * along the Morton order.
 *
 * Same quantisation, arguments, outputs, workspace and errors as
 * tess_hilbert_sort; the key is the plain bit interleave of the three grid
 * coordinates (most significant level first, x's bit first in each level)
 * instead of the Hilbert index.  Use the workspace size of
 * tess_hilbert_sort_workspace(n).
 * ------------------------------------------------------------------------- */
tess_status tess_morton_sort(const float* pos, int n, tess_box box, int bits,
                             void* ws, size_t ws_bytes,
                             int32_t* perm, uint32_t* keys_sorted, float* pos_sorted,
                             int32_t* dev_status, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Allocation-free Hilbert sort.  The paper has no counterpart: this is a
 * library convenience.
 *
 * Same computation, arguments and outputs as tess_hilbert_sort, but without a
 * workspace argument: the scratch memory is an array inside the library
 * (device memory, TESS_HILBERT_SORT_STATIC_BYTES = 21 MiB, held by every GPU
 * that loads the library until the process exits).  It is meant for callers
 * that cannot allocate device
 * memory -- for example a plugin whose host program owns all device buffers,
 * or a time-step loop that must not call cudaMalloc because it synchronises
 * the device -- and that have no buffer to lend as a workspace.
 *
 *   n  1 .. TESS_HILBERT_SORT_STATIC_MAX_N; larger n returns
 *      TESS_ERR_TOO_LARGE (use tess_hilbert_sort with a workspace instead)
 *
 * Each call looks up the array's device address in the current context (a
 * host-side query, so a context destroyed and created again never receives
 * a stale address); the first call in a context may load the library's
 * device code, so make it before any stream capture.  All calls
 * on a device share the array: calls that overlap on the GPU (different
 * streams, or unordered host threads) race on it and corrupt each other's
 * results, so order them on one stream.  Each call clears what must start at
 * zero; nothing else carries over between calls.
 * Errors: those of tess_hilbert_sort, plus TOO_LARGE.
 * ------------------------------------------------------------------------- */
#define TESS_HILBERT_SORT_STATIC_MAX_N (1 << 20)
#define TESS_HILBERT_SORT_STATIC_BYTES (21u << 20)   /* >= tess_hilbert_sort_workspace(MAX_N) */
tess_status tess_hilbert_sort_static(const float* pos, int n, tess_box box, int bits,
                                     int32_t* perm, uint32_t* keys_sorted, float* pos_sorted,
                                     int32_t* dev_status, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Verlet neighbor list at rs = rc + skin -- Tessera keeps every per-atom
 * shape constant from one rebuild to the next and names a neighbor search
 * in three levels (Tessera, abstract).
 *
 * Row i lists every j != i whose minimum-image distance to i is below rs
 * (strictly), computed in fp32.  The list is full (j in row i iff i in row
 * j) and lives in the index space of `pos` (pass the Hilbert-sorted
 * positions for locality; any order gives the same sets).  Within a row
 * the order is unspecified but deterministic for a given input.
 *
 *   pos            [n,4] float (x, y, z, ignored), 16-byte aligned
 *   rc, skin       cutoff and skin (rc > 0, skin >= 0); rs = rc + skin in fp32
 *   max_neighbors  row capacity cap >= 1
 *   flags          0, or'ed TESS_NO_PAD_FILL and at most one of
 *                  TESS_LANE2_SEARCH, TESS_LANE_SEARCH, TESS_TILE_SEARCH
 *                  (three search kernels: the same lists in other orders
 *                  within rows; none named picks the library's default, and
 *                  boxes shorter than 2 rs + 2e-3 always take the tile
 *                  search)
 *   ws, ws_bytes   scratch of at least tess_build_neighbors_workspace(...)
 *   nbr            [n, cap] int32 out: row i in nbr[i*cap .. i*cap+cap);
 *                  the first min(counts[i], cap) slots hold neighbors, the
 *                  rest are -1 (not written under TESS_NO_PAD_FILL)
 *   counts         [n] int32 out: TRUE neighbor count (may exceed cap; then
 *                  which cap neighbors are stored is unspecified)
 *   overflow       [1] int32 out: 0, or TESS_DEV_OVERFLOW if any count > cap,
 *                  or'ed with TESS_DEV_BAD_INPUT if a position is outside
 *                  [0, L) or not finite (its list is then unspecified), and
 *                  with TESS_DEV_TIMEOUT if the cell-offset scan's wait
 *                  between blocks gave up (every output is then invalid)
 * Errors: INVALID_ARG, BOX_TOO_SMALL (some L_d < 2 * rs, where the minimum
 * image is not unique), WORKSPACE_TOO_SMALL, CUDA.
 * ------------------------------------------------------------------------- */
size_t tess_build_neighbors_workspace(int n, tess_box box, float rc, float skin);
tess_status tess_build_neighbors(const float* pos, int n, tess_box box, float rc, float skin,
                                 int max_neighbors, int flags, void* ws, size_t ws_bytes,
                                 int32_t* nbr, int32_t* counts, int32_t* overflow,
                                 tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Skin check -- Tessera's conservative skin keeps the neighbor graph valid
 * while atoms move between rebuilds (Tessera, abstract).  Rebuild when some atom has moved more than
 * skin/2 since the reference frame: max_i |minimg(r_i - r_i^ref)|^2 >
 * (skin/2)^2.  Displacements, squares and the threshold are fp64 (each
 * operation one IEEE rounding: (dx*dx + dy*dy) + dz*dz), so the flag and
 * the maximum are exact functions of the fp32 inputs.
 *
 *   pos, pos_ref  [n,4] float, same index order, 16-byte aligned
 *   rebuild       [1] int32 out: 1 to rebuild, else 0
 *   max_disp2     [1] double out, nullable: the maximum squared displacement
 * Errors: INVALID_ARG (n <= 0, null, skin < 0, misaligned), CUDA.
 * ------------------------------------------------------------------------- */
tess_status tess_skin_check(const float* pos, const float* pos_ref, int n, tess_box box, float skin,
                            int32_t* rebuild, double* max_disp2, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Edge geometry and one-hop aggregation -- each message-passing layer
 * aggregates one-hop neighbor features within the cutoff (review of arXiv
 * 2505.06711, "load-bearing attack" paragraph); Tessera fuses such kernels
 * (Tessera, abstract).
 *
 * For row i and each of its first min(counts[i], cap) listed j (entries < 0
 * skipped): r_ij = minimg(r_j - r_i), r = |r_ij|, f_c(r) = (cos(pi r / rc) +
 * 1) / 2 for r < rc else 0, unit = r_ij / r (0 if r = 0), and
 *     out[i, f] = sum_j f_c(r_ij) * feat[j, f]       (fp32 accumulation)
 *
 *   pos          [n,4] float, 16-byte aligned
 *   nbr, counts  the list from tess_build_neighbors (cap = max_neighbors)
 *   feat         [n, F] float, row-major;  out  [n, F] float
 *   edge_vec     [n, cap, 4] float out, nullable: (rx, ry, rz, r)
 *   edge_fc      [n, cap] float out, nullable: f_c
 *   edge_unit    [n, cap, 4] float out, nullable: (ux, uy, uz, 0)
 *   Unused slots of the edge arrays are written 0.
 * Errors: INVALID_ARG (n <= 0, F < 1, cap < 1, rc <= 0, null, misaligned),
 * BOX_TOO_SMALL (some L_d < 2 rc), CUDA.
 * ------------------------------------------------------------------------- */
tess_status tess_edge_aggregate(const float* pos, int n, tess_box box, float rc,
                                const int32_t* nbr, const int32_t* counts, int max_neighbors,
                                const float* feat, int F, float* out,
                                float* edge_vec, float* edge_fc, float* edge_unit,
                                tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Backward of the aggregation -- in Tessera the backward pass that yields
 * the forces goes through the same neighbor exchange again (Tessera,
 * abstract); the review of arXiv 2505.06711 describes the same
 * vector-Jacobian product over one-hop edges.
 *
 * Given g = dL/d out ([n, F]), writes
 *   grad_feat[i] = dL/d feat[i] = sum_{j in row i} f_c(r_ij) g_j
 *   grad_pos[i]  = dL/d r_i     = -sum_{j in row i} f_c'(r_ij) (g_i . h_j + g_j . h_i) r_ij / |r_ij|
 * (f_c' = d f_c / d r; edges with r >= rc contribute nothing).  These are
 * the chain rule of tess_edge_aggregate for a FULL SYMMETRIC list without
 * overflow (j in row i exactly when i in row j), which is what
 * tess_build_neighbors writes when its overflow word is 0; the symmetry
 * lets every row gather its own gradients.  The forces of a model layer are
 * -grad_pos.
 *
 *   feat, grad_out  [n, F] float, 16-byte aligned, F = 4 * 2^k (4 ... 256)
 *   grad_feat       [n, F] float out, 16-byte aligned
 *   grad_pos        [n, 3] float out
 *   max_neighbors   <= 512
 * Errors: INVALID_ARG (as tess_edge_aggregate, plus F or cap outside the
 * supported set, misaligned feature arrays), BOX_TOO_SMALL, CUDA.
 * ------------------------------------------------------------------------- */
tess_status tess_edge_aggregate_backward(const float* pos, int n, tess_box box, float rc,
                                         const int32_t* nbr, const int32_t* counts, int max_neighbors,
                                         const float* feat, const float* grad_out, int F,
                                         float* grad_feat, float* grad_pos, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Closest listed pair -- a structural check for atoms that come anomalously
 * close (Tessera's runs were checked for such pairs; Tessera, abstract).
 *
 * Over every listed (i, j) -- the first min(counts[i], max_neighbors)
 * entries of row i, entries < 0 or >= n skipped -- the smallest squared
 * minimum-image distance and the pair that has it.  Distances are computed
 * as tess_skin_check computes displacements: fp64 from the fp32
 * coordinates, one IEEE rounding per product and sum, (dx^2 + dy^2) + dz^2.
 * Ties go to the smallest i, then the smallest j.  Reads the list once
 * (about 4 bytes per listed pair), so it is meant for occasional checks.
 *
 *   pos      [n, 4] float (sorted index space, as the list), 16-byte aligned
 *   ws       tess_min_pair_distance_workspace() bytes, 16-byte aligned,
 *            nothing needs to be zeroed
 *   min_r2   [1] double out: the smallest r^2, +infinity if nothing is listed
 *   min_pair [2] int32 out: (i, j), or (-1, -1) if nothing is listed
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL, CUDA.
 * ------------------------------------------------------------------------- */
size_t tess_min_pair_distance_workspace(void);
tess_status tess_min_pair_distance(const float* pos, int n, tess_box box, const int32_t* nbr,
                                   const int32_t* counts, int max_neighbors, void* ws, size_t ws_bytes,
                                   double* min_r2, int32_t* min_pair, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step graph -- one time step as a CUDA graph whose rebuild branch is taken
 * on the device.  Tessera replays each interval between rebuilds as one CUDA
 * graph (Tessera, abstract); here the skin check's flag sets the condition
 * of a conditional (IF) node, so a loop of launches needs no host round trip
 * per step, rebuilds included.  One launch:
 *   pos_cur = pos gathered into the order of the last rebuild (perm)
 *   skin check of pos_cur against pos_sorted -> *rebuild, *max_disp2
 *   rebuild = flag, or a pending request (control[0], then cleared);
 *             control[1] counts rebuilds
 *   IF rebuild: tess_hilbert_sort(pos) -> perm, keys, pos_sorted;
 *               tess_build_neighbors(pos_sorted) -> nbr, counts, overflow;
 *               pos_cur = pos_sorted
 *   tess_edge_aggregate(pos_cur, nbr, counts, feat) -> out
 * The caller writes the step's positions into `pos` (original index order)
 * before each launch.  `feat` is read in the index order of the current
 * sort: a caller whose features follow the atoms re-orders them after a
 * launch whose *rebuild is 1 (perm gives the order).  Every buffer is
 * device memory owned by the caller and must outlive the graph; sizes as for
 * the entry points above.  The first launch after create always rebuilds.
 * ------------------------------------------------------------------------- */
typedef struct tess_step_buffers {
    int n;                 /* atoms */
    tess_box box;
    float rc, skin;
    int max_neighbors;     /* list capacity per row */
    int bits;              /* Hilbert grid bits, 1..10 */
    int F;                 /* features per atom */
    int flags;             /* tess_build_neighbors flags */
    const float* pos;      /* [n, 3] current positions, original order (written by the caller) */
    const float* feat;     /* [n, F] */
    void* ws_sort;         /* tess_hilbert_sort_workspace(n) bytes, 256-byte aligned */
    size_t ws_sort_bytes;
    void* ws_list;         /* tess_build_neighbors_workspace(...) bytes, 256-byte aligned */
    size_t ws_list_bytes;
    int32_t* perm;         /* [n] */
    uint32_t* keys;        /* [n] */
    float* pos_sorted;     /* [n, 4] positions at the last rebuild, sorted order */
    float* pos_cur;        /* [n, 4] current positions, sorted order */
    int32_t* nbr;          /* [n, max_neighbors] */
    int32_t* counts;       /* [n] */
    int32_t* overflow;     /* [1] */
    int32_t* sort_status;  /* [1] */
    int32_t* rebuild;      /* [1] out: 1 when the step rebuilt */
    double* max_disp2;     /* [1] out */
    int32_t* control;      /* [2] device words (see above) */
    float* out;            /* [n, F] */
} tess_step_buffers;

typedef struct tess_step_graph tess_step_graph;

/* Builds and instantiates the graph (stream capture on `stream`, which must
 * not be the legacy default stream) and queues a rebuild request for the
 * first launch.  Call outside any other capture, with stage timing off or on
 * (timing is skipped while capturing).  Errors: INVALID_ARG,
 * WORKSPACE_TOO_SMALL, BOX_TOO_SMALL, CUDA (e.g. a driver without
 * conditional nodes); *out is NULL then. */
tess_status tess_step_graph_create(const tess_step_buffers* b, tess_stream_t stream, tess_step_graph** out);
/* One step: cudaGraphLaunch on `stream`. */
tess_status tess_step_graph_launch(tess_step_graph* g, tess_stream_t stream);
/* Makes the next launch rebuild whatever the skin check says (stream-ordered). */
tess_status tess_step_graph_request_rebuild(const tess_step_buffers* b, tess_stream_t stream);
void tess_step_graph_destroy(tess_step_graph* g);

/* ---------------------------------------------------------------------------
 * Look-back timeout probe (diagnostic, no counterpart in the paper).  The
 * sort's counting passes wait on each other through a decoupled look-back
 * whose wait is bounded: after a fixed number of polls it gives up, sets
 * TESS_DEV_TIMEOUT in the status word and lets the kernel finish, so the
 * GPU context stays usable.  This call makes that happen on purpose: one
 * block runs the second tile of a pass whose first tile never runs.  It
 * takes a few seconds, writes only inside `ws`, and its output means
 * nothing; *dev_status ends with TESS_DEV_TIMEOUT set.
 *   ws  tess_debug_lookback_timeout_workspace() bytes, 256-byte aligned
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL, CUDA.
 * ------------------------------------------------------------------------- */
size_t tess_debug_lookback_timeout_workspace(void);
tess_status tess_debug_lookback_timeout(void* ws, size_t ws_bytes, int32_t* dev_status, tess_stream_t stream);

/* ---------------------------------------------------------------------------
 * Stage timing (diagnostic).  When enabled, each entry point records CUDA
 * events on its stream around its kernels; tess_stage_times adds the elapsed
 * times of all recorded calls per stage (this synchronises on the events)
 * and clears them.  Stages: 0 space-filling-curve keys, 1 key sort, 2 cell
 * binning, 3 pair search, 4 skin check, 5 edge aggregate, 6 aggregate backward,
 * 7 incremental re-sort (its fallback full sort records under 0 and 1),
 * 8 closest listed pair.  Returns the number of
 * stages written (<= max_stages).  ms_out[k] = total milliseconds,
 * calls_out[k] (nullable) = number of timed calls.  The events are kept in a
 * process-wide pool and reused: after one timed round has been read back, a
 * second round records without creating events.  The pool, the records and
 * the on/off switch are the library's only process state (a mutex guards
 * them); stage timing is off unless enabled.
 * ------------------------------------------------------------------------- */
void tess_stage_timing(int enable);
int tess_stage_times(double* ms_out, long long* calls_out, int max_stages);

#ifdef __cplusplus
}
#endif
#endif /* TESS_H */
