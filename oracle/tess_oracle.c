/*
 * tess_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * neighbor-rebuild path (Hilbert sort, Verlet list, skin check, one-hop
 * cosine-cutoff aggregation).
 *
 * TEST INFRASTRUCTURE ONLY.  The product library never links, loads or
 * calls this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no source, header, table or constant
 * generator with the CUDA library: both sides were written separately from
 * the same definitions.
 *
 * What the method computes comes from "Ab Initio Accuracy Beyond the
 * Cutoff: Distributed Message-Passing Equivariant Attention at
 * Tens-of-Millions-of-Atom Scale" (Tessera), abstract: atoms are sorted
 * along a space-filling curve, a conservative neighbor skin keeps the
 * topology valid between rebuilds, shapes stay fixed between rebuilds, and
 * each message-passing layer consumes one-hop neighbor features.  The
 * one-hop semantics (aggregate only neighbors within the original cutoff)
 * is stated in the review of arXiv 2505.06711 (ghost-atom message passing),
 * "load-bearing attack" paragraph.  The pages fix no formula; every choice
 * the pages leave open is marked READING below.
 *
 * Precision: all distances, displacements and sums are fp64 computed from
 * the fp32 inputs.  The single decision taken in fp32 is the Hilbert grid
 * quantisation (an integer decided by floating point), which the GPU path
 * takes in fp32 too.  Build with -O2 -ffp-contract=off (no FMA contraction,
 * no fast-math) so every operation is one IEEE rounding in source order.
 *
 * Parity pins (tests under tests/): Hilbert bijection, unit steps, nesting
 * and a hand-derived 1-bit table; brute force == cell list; pair symmetry;
 * hand 2-atom and 4-atom periodic examples; skin hand cases; cutoff closed
 * forms and aggregate identities.  No function here is parity-unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* pi to double precision (not every libc exposes M_PI under -std=c11) */
#define ORACLE_PI 3.14159265358979323846

/* ------------------------------------------------------------------------ */
/* threads                                                                  */
/* ------------------------------------------------------------------------ */

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* C1. Hilbert key                                                          */
/* ------------------------------------------------------------------------ */

/*
 * Grid quantisation of one coordinate (READING: the pages name no grid).
 * The scale is one fp32 IEEE division 2^bits / L, the product x*scale is one
 * fp32 multiply rounded to nearest, then floor and clamp into [0, 2^bits-1].
 * Products below 1 (including negative values and NaN) give cell 0.
 */
uint32_t oracle_quantize(float x, float L, int bits)
{
    float scale = (float)(1u << bits) / L;
    float prod = x * scale;
    uint32_t top = (1u << bits) - 1u;
    if (!(prod >= 1.0f)) return 0u;
    float fl = floorf(prod);
    if (fl >= (float)top) return top;
    return (uint32_t)fl;
}

/*
 * 3-D Hilbert index of grid point (q0, q1, q2), each in [0, 2^bits).
 * Published method: J. Skilling, "Programming the Hilbert curve", AIP Conf.
 * Proc. 707 (2004) -- the axes-to-transpose transform followed by reading
 * the transposed words out most-significant level first.  Axis 0 is x.
 * READING: the pages never name the Hilbert variant, the bit width or the
 * axis order; Skilling's transform with x as axis 0 is the plainest choice.
 */
uint32_t oracle_hilbert_index(uint32_t q0, uint32_t q1, uint32_t q2, int bits)
{
    uint32_t X[3] = {q0, q1, q2};
    uint32_t top_bit = 1u << (bits - 1);

    /* Walk the levels from the coarsest down.  At level Q, for each axis i:
     * if axis i has bit Q set, flip the lower bits of axis 0; otherwise swap
     * the lower bits of axis 0 and axis i.  This undoes the rotations and
     * reflections of the sub-cubes above the current level. */
    for (uint32_t Q = top_bit; Q > 1u; Q >>= 1) {
        uint32_t low = Q - 1u;
        for (int i = 0; i < 3; ++i) {
            if (X[i] & Q) {
                X[0] ^= low;
            } else {
                uint32_t diff = (X[0] ^ X[i]) & low;
                X[0] ^= diff;
                X[i] ^= diff;
            }
        }
    }

    /* Gray-encode across the axes. */
    X[1] ^= X[0];
    X[2] ^= X[1];

    /* Fold the parity of the last axis into every axis. */
    uint32_t fold = 0u;
    for (uint32_t Q = top_bit; Q > 1u; Q >>= 1) {
        if (X[2] & Q) fold ^= Q - 1u;
    }
    for (int i = 0; i < 3; ++i) X[i] ^= fold;

    /* Read the transposed form out: level by level from the most
     * significant, axis 0's bit first within each level. */
    uint32_t key = 0u;
    for (int level = bits - 1; level >= 0; --level) {
        for (int i = 0; i < 3; ++i) {
            key = (key << 1) | ((X[i] >> level) & 1u);
        }
    }
    return key;
}

static int cmp_u64(const void* a, const void* b)
{
    uint64_t x = *(const uint64_t*)a, y = *(const uint64_t*)b;
    return (x > y) - (x < y);
}

/*
 * Morton (Z-order) index of grid point (q0, q1, q2): the bits of the three
 * coordinates interleaved most-significant level first, axis 0's bit first
 * within each level -- the same read-out as the Hilbert index without the
 * transform.  The Tessera abstract compares its curve against this order
 * (neighbor-search cost grows 3.0x along it, 1.7x along its own curve).
 */
uint32_t oracle_morton_index(uint32_t q0, uint32_t q1, uint32_t q2, int bits)
{
    const uint32_t X[3] = {q0, q1, q2};
    uint32_t key = 0u;
    for (int level = bits - 1; level >= 0; --level)
        for (int i = 0; i < 3; ++i) key = (key << 1) | ((X[i] >> level) & 1u);
    return key;
}

void oracle_morton_index_many(const uint32_t* q, int64_t m, int bits, uint32_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < m; ++k) out[k] = oracle_morton_index(q[3 * k], q[3 * k + 1], q[3 * k + 2], bits);
}

/* Stable sort by Morton key (same contract as oracle_hilbert_sort). */
void oracle_morton_sort(const float* pos, int stride, int64_t n, const float* L, int bits, int32_t* perm,
                        uint32_t* keys_sorted)
{
    uint64_t* kv = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)(n > 0 ? n : 1));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float* p = pos + i * stride;
        uint32_t key = oracle_morton_index(oracle_quantize(p[0], L[0], bits), oracle_quantize(p[1], L[1], bits),
                                           oracle_quantize(p[2], L[2], bits), bits);
        kv[i] = ((uint64_t)key << 32) | (uint64_t)(uint32_t)i;
    }
    qsort(kv, (size_t)n, sizeof(uint64_t), cmp_u64);
    for (int64_t k = 0; k < n; ++k) {
        perm[k] = (int32_t)(uint32_t)(kv[k] & 0xffffffffu);
        if (keys_sorted) keys_sorted[k] = (uint32_t)(kv[k] >> 32);
    }
    free(kv);
}

/* Hilbert indices of m integer grid points q[m][3]. */
void oracle_hilbert_index_many(const uint32_t* q, int64_t m, int bits, uint32_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < m; ++k) out[k] = oracle_hilbert_index(q[3 * k], q[3 * k + 1], q[3 * k + 2], bits);
}

/* Keys of n positions (row stride `stride` floats, x y z first). */
void oracle_hilbert_keys(const float* pos, int stride, int64_t n, const float* L,
                         int bits, uint32_t* keys)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float* p = pos + i * stride;
        uint32_t qx = oracle_quantize(p[0], L[0], bits);
        uint32_t qy = oracle_quantize(p[1], L[1], bits);
        uint32_t qz = oracle_quantize(p[2], L[2], bits);
        keys[i] = oracle_hilbert_index(qx, qy, qz, bits);
    }
}

/*
 * C2. Permutation: order atoms by key, ties by ascending input index
 * (READING: the tie-break is unstated; stable-by-index makes the order
 * total, so perm is unique).  perm[k] = input index of the atom at rank k.
 */
void oracle_hilbert_sort(const float* pos, int stride, int64_t n, const float* L,
                         int bits, int32_t* perm, uint32_t* keys_sorted)
{
    uint32_t* keys = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)(n > 0 ? n : 1));
    uint64_t* kv = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)(n > 0 ? n : 1));
    oracle_hilbert_keys(pos, stride, n, L, bits, keys);
    for (int64_t i = 0; i < n; ++i) kv[i] = ((uint64_t)keys[i] << 32) | (uint64_t)(uint32_t)i;
    qsort(kv, (size_t)n, sizeof(uint64_t), cmp_u64);
    for (int64_t k = 0; k < n; ++k) {
        perm[k] = (int32_t)(uint32_t)(kv[k] & 0xffffffffu);
        if (keys_sorted) keys_sorted[k] = (uint32_t)(kv[k] >> 32);
    }
    free(kv);
    free(keys);
}

/* ------------------------------------------------------------------------ */
/* C3. Verlet list at rs = rc + skin, full, self excluded, minimum image     */
/* ------------------------------------------------------------------------ */

/* Minimum-image component in fp64 (READING: orthorhombic box with origin 0;
 * a component beyond half a box length is brought back by one length). */
static double min_image(double d, double L)
{
    if (d > 0.5 * L) return d - L;
    if (d < -0.5 * L) return d + L;
    return d;
}

/* Squared minimum-image distance from atom i to atom j, fp64. */
static double pair_r2(const float* pi, const float* pj, const double Ld[3])
{
    double dx = min_image((double)pj[0] - (double)pi[0], Ld[0]);
    double dy = min_image((double)pj[1] - (double)pi[1], Ld[1]);
    double dz = min_image((double)pj[2] - (double)pi[2], Ld[2]);
    return dx * dx + dy * dy + dz * dz;
}

static int cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Brute force O(n^2).  Row i of nbr ([n, cap], -1 pads) holds its neighbors
 * in ascending index order; counts[i] is the true count, which may exceed
 * cap (then the row holds the cap smallest indices).  Accept iff
 * r^2 < rs^2 strictly, rs = rc + skin in fp64 (READING: strict inequality and
 * a list radius of exactly rc + skin).  Returns 1 if any count > cap.
 */
int oracle_neighbors_brute(const float* pos, int stride, int64_t n, const float* L,
                           float rc, float skin, int cap, int32_t* nbr, int32_t* counts)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    const double rs = (double)rc + (double)skin;
    const double rs2 = rs * rs;
    int overflow = 0;

    #pragma omp parallel for schedule(dynamic, 64) reduction(|:overflow)
    for (int64_t i = 0; i < n; ++i) {
        int32_t* row = nbr + i * (int64_t)cap;
        int32_t cnt = 0;
        for (int c = 0; c < cap; ++c) row[c] = -1;
        for (int64_t j = 0; j < n; ++j) {
            if (j == i) continue;
            if (pair_r2(pos + i * stride, pos + j * stride, Ld) < rs2) {
                if (cnt < cap) row[cnt] = (int32_t)j;
                ++cnt;
            }
        }
        counts[i] = cnt;
        if (cnt > cap) overflow = 1;
    }
    return overflow;
}

/*
 * Straightforward cell list: ncell_d = floor(L_d / (rs * 1.0001)) cells per
 * axis, each atom in the cell floor(x / w_d) (clamped into the grid), and the
 * 27 cells around an atom's own cell searched with the same fp64 test as the
 * brute force.  With at least 3 cells per axis the 27 cells are distinct.
 * Falls back to the brute force when an axis has fewer than 3 cells.
 * Same output contract as oracle_neighbors_brute.
 */
int oracle_neighbors_cells(const float* pos, int stride, int64_t n, const float* L,
                           float rc, float skin, int cap, int32_t* nbr, int32_t* counts)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    const double rs = (double)rc + (double)skin;
    const double rs2 = rs * rs;
    int64_t nc[3];
    double w[3];
    for (int d = 0; d < 3; ++d) {
        nc[d] = (int64_t)floor(Ld[d] / (rs * 1.0001));
        if (nc[d] < 3) return oracle_neighbors_brute(pos, stride, n, L, rc, skin, cap, nbr, counts);
        w[d] = Ld[d] / (double)nc[d];
    }
    const int64_t ncell = nc[0] * nc[1] * nc[2];

    /* counting sort of atoms into cells */
    int64_t* cell_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    int64_t* start = (int64_t*)calloc((size_t)ncell + 1, sizeof(int64_t));
    int64_t* fill = (int64_t*)calloc((size_t)ncell, sizeof(int64_t));
    int64_t* members = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        int64_t c3[3];
        for (int d = 0; d < 3; ++d) {
            double f = floor((double)pos[i * stride + d] / w[d]);
            int64_t c = (f < 0.0 || f != f) ? 0 : (int64_t)f;
            if (c >= nc[d]) c = nc[d] - 1;
            c3[d] = c;
        }
        cell_of[i] = (c3[2] * nc[1] + c3[1]) * nc[0] + c3[0];
        start[cell_of[i] + 1]++;
    }
    for (int64_t c = 0; c < ncell; ++c) start[c + 1] += start[c];
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = cell_of[i];
        members[start[c] + fill[c]++] = i;   /* ascending i within a cell */
    }

    int overflow = 0;
    #pragma omp parallel reduction(|:overflow)
    {
        int64_t bufcap = 1024;
        int32_t* buf = (int32_t*)malloc(sizeof(int32_t) * (size_t)bufcap);
        #pragma omp for schedule(dynamic, 256)
        for (int64_t i = 0; i < n; ++i) {
            int64_t c = cell_of[i];
            int64_t cx = c % nc[0], cy = (c / nc[0]) % nc[1], cz = c / (nc[0] * nc[1]);
            int64_t cnt = 0;
            for (int dz = -1; dz <= 1; ++dz)
            for (int dy = -1; dy <= 1; ++dy)
            for (int dx = -1; dx <= 1; ++dx) {
                int64_t x = (cx + dx + nc[0]) % nc[0];
                int64_t y = (cy + dy + nc[1]) % nc[1];
                int64_t z = (cz + dz + nc[2]) % nc[2];
                int64_t cc = (z * nc[1] + y) * nc[0] + x;
                for (int64_t k = start[cc]; k < start[cc + 1]; ++k) {
                    int64_t j = members[k];
                    if (j == i) continue;
                    if (pair_r2(pos + i * stride, pos + j * stride, Ld) < rs2) {
                        if (cnt == bufcap) {
                            bufcap *= 2;
                            buf = (int32_t*)realloc(buf, sizeof(int32_t) * (size_t)bufcap);
                        }
                        buf[cnt++] = (int32_t)j;
                    }
                }
            }
            qsort(buf, (size_t)cnt, sizeof(int32_t), cmp_i32);
            int32_t* row = nbr + i * (int64_t)cap;
            for (int s = 0; s < cap; ++s) row[s] = (s < cnt) ? buf[s] : -1;
            counts[i] = (int32_t)cnt;
            if (cnt > cap) overflow = 1;
        }
        free(buf);
    }
    free(members);
    free(fill);
    free(start);
    free(cell_of);
    return overflow;
}

/*
 * One row of the list, brute force over all n atoms, for sampled checks on
 * large systems.  Writes up to max_out ascending indices, returns the count.
 */
int64_t oracle_neighbors_of(const float* pos, int stride, int64_t n, const float* L,
                            float rc, float skin, int64_t i, int32_t* out, int64_t max_out)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    const double rs = (double)rc + (double)skin;
    const double rs2 = rs * rs;
    int64_t cnt = 0;
    for (int64_t j = 0; j < n; ++j) {
        if (j == i) continue;
        if (pair_r2(pos + i * stride, pos + j * stride, Ld) < rs2) {
            if (cnt < max_out) out[cnt] = (int32_t)j;
            ++cnt;
        }
    }
    return cnt;
}

/*
 * Rows rows[0..m) of the list by brute force over all n atoms (sampled
 * checks on large systems), rows in parallel.  Same row contract as the
 * full-list functions: ascending indices, -1 pads, true counts.
 */
void oracle_neighbors_rows(const float* pos, int stride, int64_t n, const float* L, float rc, float skin,
                           const int64_t* rows, int64_t m, int cap, int32_t* nbr, int32_t* counts)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    const double rs = (double)rc + (double)skin;
    const double rs2 = rs * rs;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < m; ++k) {
        const int64_t i = rows[k];
        int32_t* row = nbr + k * (int64_t)cap;
        int32_t cnt = 0;
        for (int c = 0; c < cap; ++c) row[c] = -1;
        for (int64_t j = 0; j < n; ++j) {
            if (j == i) continue;
            if (pair_r2(pos + i * stride, pos + j * stride, Ld) < rs2) {
                if (cnt < cap) row[cnt] = (int32_t)j;
                ++cnt;
            }
        }
        counts[k] = cnt;
    }
}

/*
 * Pair distances in fp64 for a list of (i, j) pairs -- used by tests to find
 * pairs whose distance is within a band of rs, where an fp32 test may round
 * either way.
 */
void oracle_pair_distances(const float* pos, int stride, const float* L,
                           const int32_t* pi, const int32_t* pj, int64_t m, double* dist)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < m; ++k) {
        dist[k] = sqrt(pair_r2(pos + (int64_t)pi[k] * stride, pos + (int64_t)pj[k] * stride, Ld));
    }
}

/* ------------------------------------------------------------------------ */
/* C4. Skin check                                                            */
/* ------------------------------------------------------------------------ */

/*
 * Squared minimum-image displacement of every atom from its reference
 * position, fp64, in the order (dx*dx + dy*dy) + dz*dz; the flag is
 * max_i disp2_i > (skin/2)^2 with skin/2 and its square in fp64.
 * READING: "conservative neighbor skin" is the standard criterion -- no atom
 * has moved more than half the skin since the last rebuild -- which
 * guarantees that no pair closer than rc can have been missing from a list
 * built at rc + skin.  Returns the flag; *max_d2 receives the maximum.
 */
int oracle_skin_check(const float* pos, const float* ref, int stride, int64_t n,
                      const float* L, float skin, double* max_d2)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    const double half = 0.5 * (double)skin;
    const double h2 = half * half;
    double m = 0.0;
    #pragma omp parallel for schedule(static) reduction(max:m)
    for (int64_t i = 0; i < n; ++i) {
        const float* p = pos + i * stride;
        const float* r = ref + i * stride;
        double dx = min_image((double)p[0] - (double)r[0], Ld[0]);
        double dy = min_image((double)p[1] - (double)r[1], Ld[1]);
        double dz = min_image((double)p[2] - (double)r[2], Ld[2]);
        double d2 = dx * dx + dy * dy + dz * dz;
        if (d2 > m) m = d2;
    }
    if (max_d2) *max_d2 = m;
    return m > h2 ? 1 : 0;
}

/* ------------------------------------------------------------------------ */
/* C5. Edge geometry and one-hop aggregation                                 */
/* ------------------------------------------------------------------------ */

/*
 * Smooth cosine cutoff, READING of "smooth cosine cutoff": the Behler form
 * f_c(r) = (cos(pi r / rc) + 1) / 2 for r < rc, and 0 beyond.
 */
double oracle_cutoff(double r, double rc)
{
    if (r < rc) return 0.5 * (cos(ORACLE_PI * r / rc) + 1.0);
    return 0.0;
}

double oracle_cutoff(double r, double rc);

/* C5 for rows rows[0..m) only (sampled checks): out/out_abs are [m, F]. */
void oracle_edge_aggregate_rows(const float* pos, int stride, int64_t n, const float* L, float rc,
                                const int32_t* nbr, const int32_t* counts, int cap, const float* feat, int F,
                                const int64_t* rows, int64_t m, double* out, double* out_abs)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t k = 0; k < m; ++k) {
        const int64_t i = rows[k];
        double* o = out + k * (int64_t)F;
        double* oa = out_abs + k * (int64_t)F;
        for (int f = 0; f < F; ++f) { o[f] = 0.0; oa[f] = 0.0; }
        int64_t mm = counts[i] < cap ? counts[i] : cap;
        for (int64_t s = 0; s < mm; ++s) {
            int32_t j = nbr[i * (int64_t)cap + s];
            if (j < 0 || j >= n) continue;
            const float* pi = pos + i * stride;
            const float* pj = pos + (int64_t)j * stride;
            double dx = min_image((double)pj[0] - (double)pi[0], Ld[0]);
            double dy = min_image((double)pj[1] - (double)pi[1], Ld[1]);
            double dz = min_image((double)pj[2] - (double)pi[2], Ld[2]);
            double fc = oracle_cutoff(sqrt(dx * dx + dy * dy + dz * dz), (double)rc);
            if (fc == 0.0) continue;
            const float* h = feat + (int64_t)j * F;
            for (int f = 0; f < F; ++f) {
                o[f] += fc * (double)h[f];
                oa[f] += fc * fabs((double)h[f]);
            }
        }
    }
}

/*
 * For every row i and each listed j (the first min(counts[i], cap) slots,
 * negative entries skipped): r_ij = minimum image of (r_j - r_i) (READING:
 * the vector points from i to j), |r_ij|, f_c(|r_ij|), unit = r_ij/|r_ij|
 * (0 when |r_ij| = 0), and out_i[f] = sum_j f_c(|r_ij|) h_j[f] accumulated in
 * fp64 (READING: a plain sum, no normalisation, no self term).  out_abs
 * receives sum_j f_c |h_j[f]|, the conditioning of each sum.  Edge arrays
 * (nullable) are [n, cap, 4] for (rx, ry, rz, |r|), [n, cap] for f_c and
 * [n, cap, 4] for (ux, uy, uz, 0); unused slots are 0.
 */
void oracle_edge_aggregate(const float* pos, int stride, int64_t n, const float* L,
                           float rc, const int32_t* nbr, const int32_t* counts, int cap,
                           const float* feat, int F, double* out, double* out_abs,
                           double* edge_vec, double* edge_fc, double* edge_unit)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        double* o = out + i * (int64_t)F;
        double* oa = out_abs ? out_abs + i * (int64_t)F : NULL;
        for (int f = 0; f < F; ++f) { o[f] = 0.0; if (oa) oa[f] = 0.0; }
        int64_t m = counts[i] < cap ? counts[i] : cap;
        if (m < 0) m = 0;
        for (int s = 0; s < cap; ++s) {
            int64_t e = i * (int64_t)cap + s;
            if (edge_vec) { edge_vec[4 * e] = edge_vec[4 * e + 1] = edge_vec[4 * e + 2] = edge_vec[4 * e + 3] = 0.0; }
            if (edge_fc) edge_fc[e] = 0.0;
            if (edge_unit) { edge_unit[4 * e] = edge_unit[4 * e + 1] = edge_unit[4 * e + 2] = edge_unit[4 * e + 3] = 0.0; }
            if (s >= m) continue;
            int32_t j = nbr[e];
            if (j < 0 || j >= n) continue;
            const float* pi = pos + i * stride;
            const float* pj = pos + (int64_t)j * stride;
            double dx = min_image((double)pj[0] - (double)pi[0], Ld[0]);
            double dy = min_image((double)pj[1] - (double)pi[1], Ld[1]);
            double dz = min_image((double)pj[2] - (double)pi[2], Ld[2]);
            double r = sqrt(dx * dx + dy * dy + dz * dz);
            double fc = oracle_cutoff(r, (double)rc);
            if (edge_vec) { edge_vec[4 * e] = dx; edge_vec[4 * e + 1] = dy; edge_vec[4 * e + 2] = dz; edge_vec[4 * e + 3] = r; }
            if (edge_fc) edge_fc[e] = fc;
            if (edge_unit && r > 0.0) {
                edge_unit[4 * e] = dx / r; edge_unit[4 * e + 1] = dy / r; edge_unit[4 * e + 2] = dz / r;
            }
            if (fc == 0.0) continue;
            const float* h = feat + (int64_t)j * F;
            for (int f = 0; f < F; ++f) {
                o[f] += fc * (double)h[f];
                if (oa) oa[f] += fc * fabs((double)h[f]);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of C5 (force path)                                               */
/* ------------------------------------------------------------------------ */

/* d f_c / d r of the Behler cutoff: -(pi / (2 rc)) sin(pi r / rc) for r < rc. */
double oracle_cutoff_deriv(double r, double rc)
{
    if (r < rc) return -0.5 * ORACLE_PI / rc * sin(ORACLE_PI * r / rc);
    return 0.0;
}

/*
 * Vector-Jacobian product of out_i = sum_{j in row i} f_c(|r_ij|) h_j with
 * respect to the features and the positions, given g = dL/d out ([n, F]).
 * The backward pass that yields the forces repeats the neighbor exchange
 * (Tessera, abstract); the review of arXiv 2505.06711 describes the same VJP over one-hop edges.
 * Plain chain rule over the listed edges, accumulated serially in fp64:
 *   grad_feat[j] += f_c(r_ij) g_i                       for each listed (i, j)
 *   s = f_c'(r_ij) (g_i . h_j);  grad_pos[i] -= s u_ij;  grad_pos[j] += s u_ij
 * with u_ij = r_ij / |r_ij| (0 when |r_ij| = 0).  grad_feat [n, F] and
 * grad_pos [n, 3] are overwritten.
 */
void oracle_edge_backward(const float* pos, int stride, int64_t n, const float* L, float rc,
                          const int32_t* nbr, const int32_t* counts, int cap, const float* feat,
                          const float* grad_out, int F, double* grad_feat, double* grad_pos)
{
    const double Ld[3] = {(double)L[0], (double)L[1], (double)L[2]};
    for (int64_t k = 0; k < n * (int64_t)F; ++k) grad_feat[k] = 0.0;
    for (int64_t k = 0; k < n * 3; ++k) grad_pos[k] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t m = counts[i] < cap ? counts[i] : cap;
        for (int64_t s = 0; s < m; ++s) {
            int32_t j = nbr[i * (int64_t)cap + s];
            if (j < 0 || j >= n) continue;
            const float* pi = pos + i * stride;
            const float* pj = pos + (int64_t)j * stride;
            double d[3];
            d[0] = min_image((double)pj[0] - (double)pi[0], Ld[0]);
            d[1] = min_image((double)pj[1] - (double)pi[1], Ld[1]);
            d[2] = min_image((double)pj[2] - (double)pi[2], Ld[2]);
            double r = sqrt(d[0] * d[0] + d[1] * d[1] + d[2] * d[2]);
            double fc = oracle_cutoff(r, (double)rc);
            double dfc = oracle_cutoff_deriv(r, (double)rc);
            if (fc == 0.0 && dfc == 0.0) continue;
            const float* gi = grad_out + i * (int64_t)F;
            const float* hj = feat + (int64_t)j * F;
            double dot = 0.0;
            for (int f = 0; f < F; ++f) {
                grad_feat[(int64_t)j * F + f] += fc * (double)gi[f];
                dot += (double)gi[f] * (double)hj[f];
            }
            if (r > 0.0) {
                double sc = dfc * dot / r;
                for (int a = 0; a < 3; ++a) {
                    grad_pos[i * 3 + a] -= sc * d[a];
                    grad_pos[(int64_t)j * 3 + a] += sc * d[a];
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Closest listed pair (a structural check: Tessera's runs are checked for   */
/* atoms that come anomalously close; Tessera, abstract)                     */
/* ------------------------------------------------------------------------ */

/*
 * Over every listed (i, j) -- the first min(counts[i], cap) entries of row
 * i, entries < 0 or >= n skipped -- the smallest squared minimum-image
 * distance, computed as the list computes it (pair_r2, fp64 from the fp32
 * coordinates), and the pair that has it: ties go to the smallest i, then
 * the smallest j.  No listed pair: *r2 = +infinity, *pi = *pj = -1.
 * READING: the pages only say that close pairs were looked for; the
 * closest listed pair is the plainest quantity that says whether there is
 * one.
 */
void oracle_min_pair(const float* pos, int stride, int64_t n, const float* L, const int32_t* nbr,
                     const int32_t* counts, int cap, double* r2, int32_t* pi, int32_t* pj)
{
    const double Ld[3] = {L[0], L[1], L[2]};
    double best = 1.0 / 0.0;
    int32_t bi = -1, bj = -1;
    for (int64_t i = 0; i < n; ++i) {
        int64_t m = counts[i] < cap ? counts[i] : cap;
        for (int64_t s = 0; s < m; ++s) {
            int32_t j = nbr[i * cap + s];
            if (j < 0 || j >= n) continue;
            double d = pair_r2(pos + i * stride, pos + (int64_t)j * stride, Ld);
            if (d < best || (d == best && (i < bi || (i == bi && j < bj)))) {
                best = d;
                bi = (int32_t)i;
                bj = j;
            }
        }
    }
    *r2 = best;
    *pi = bi;
    *pj = bj;
}

