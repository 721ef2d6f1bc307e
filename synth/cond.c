/*
 * cond.c -- input conditioning for the synthetic systems.
 *
 * Marks atoms that take part in a pair whose periodic distance falls in a
 * forbidden set: closer than d_min (the minimum separation of the generated
 * systems) or within +-half_width of r_band (the list radius rc + skin, so
 * that no pair sits where an fp32 distance test could round either way).
 * The higher index of each offending pair is marked; the generator then
 * re-draws those atoms.  Distances are fp64 computed from the fp32
 * coordinates that the library will actually see.
 *
 * This is part of the seeded input generator; it builds no neighbor list
 * and shares no code with the oracle or with the CUDA library.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

static double wrap_delta(double d, double L)
{
    return d - L * nearbyint(d / L);
}

/* Distance test of a against b shifted by the periodic image s. */
static inline void classify_shifted(const float* a, const float* b, const double* s, double lo2,
                                    double hi2, double dmin2, int64_t hi_idx,
                                    uint8_t* close_mark, uint8_t* band_mark)
{
    double dx = ((double)b[0] + s[0]) - (double)a[0];
    double r2 = dx * dx;
    if (r2 >= hi2 && r2 >= dmin2) return;
    double dy = ((double)b[1] + s[1]) - (double)a[1];
    r2 += dy * dy;
    if (r2 >= hi2 && r2 >= dmin2) return;
    double dz = ((double)b[2] + s[2]) - (double)a[2];
    r2 += dz * dz;
    if (r2 < dmin2) __atomic_store_n(&close_mark[hi_idx], (uint8_t)1, __ATOMIC_RELAXED);
    else if (r2 > lo2 && r2 < hi2) __atomic_store_n(&band_mark[hi_idx], (uint8_t)1, __ATOMIC_RELAXED);
}

static void classify(const float* a, const float* b, const double* L, double lo2, double hi2,
                     double dmin2, int64_t hi_idx, uint8_t* close_mark, uint8_t* band_mark)
{
    double s[3];
    for (int d = 0; d < 3; ++d) {
        double dd = (double)b[d] - (double)a[d];
        s[d] = wrap_delta(dd, L[d]) - dd;
    }
    classify_shifted(a, b, s, lo2, hi2, dmin2, hi_idx, close_mark, band_mark);
}

/* Returns the number of marked atoms (close + band). */
int64_t cond_mark(const float* pos, int64_t n, const double* L, double dmin,
                  double r_band, double half_width, uint8_t* close_mark, uint8_t* band_mark)
{
    const double lo = r_band - half_width, hi = r_band + half_width;
    const double lo2 = lo * lo, hi2 = hi * hi, dmin2 = dmin * dmin;
    double reach = hi > dmin ? hi : dmin;
    reach *= 1.000001;
    {
        /* no finer than about one atom per cell, so a short reach on a
         * sparse set does not allocate a huge grid */
        double per_atom = cbrt(L[0] * L[1] * L[2] / (double)(n > 0 ? n : 1));
        if (reach < per_atom) reach = per_atom;
    }
    int64_t g[3];
    int small = 0;
    for (int d = 0; d < 3; ++d) {
        g[d] = (int64_t)floor(L[d] / reach);
        if (g[d] < 3) small = 1;
    }
    for (int64_t i = 0; i < n; ++i) { close_mark[i] = 0; band_mark[i] = 0; }

    if (small) {
        #pragma omp parallel for schedule(dynamic, 16)
        for (int64_t i = 0; i < n; ++i)
            for (int64_t j = i + 1; j < n; ++j)
                classify(pos + 3 * i, pos + 3 * j, L, lo2, hi2, dmin2, j, close_mark, band_mark);
    } else {
        const int64_t ng = g[0] * g[1] * g[2];
        int64_t* head = (int64_t*)calloc((size_t)ng + 1, sizeof(int64_t));
        int64_t* gid = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
        int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
        for (int64_t i = 0; i < n; ++i) {
            int64_t c[3];
            for (int d = 0; d < 3; ++d) {
                double u = (double)pos[3 * i + d] / L[d];
                u -= floor(u);
                int64_t k = (int64_t)(u * (double)g[d]);
                c[d] = k < 0 ? 0 : (k >= g[d] ? g[d] - 1 : k);
            }
            gid[i] = c[0] + g[0] * (c[1] + g[1] * c[2]);
            head[gid[i] + 1]++;
        }
        for (int64_t c = 0; c < ng; ++c) head[c + 1] += head[c];
        {
            int64_t* fill = (int64_t*)calloc((size_t)ng, sizeof(int64_t));
            for (int64_t i = 0; i < n; ++i) order[head[gid[i]] + fill[gid[i]]++] = i;
            free(fill);
        }
        /* half stencil: the cell itself (pairs a<b) and 13 forward offsets */
        static const int off[13][3] = {
            {1, 0, 0}, {-1, 1, 0}, {0, 1, 0}, {1, 1, 0},
            {-1, -1, 1}, {0, -1, 1}, {1, -1, 1}, {-1, 0, 1}, {0, 0, 1}, {1, 0, 1},
            {-1, 1, 1}, {0, 1, 1}, {1, 1, 1}};
        #pragma omp parallel for schedule(dynamic, 64)
        for (int64_t c = 0; c < ng; ++c) {
            int64_t cx = c % g[0], cy = (c / g[0]) % g[1], cz = c / (g[0] * g[1]);
            const double zero[3] = {0.0, 0.0, 0.0};
            for (int64_t a = head[c]; a < head[c + 1]; ++a)
                for (int64_t b = a + 1; b < head[c + 1]; ++b) {
                    int64_t i = order[a], j = order[b];
                    /* same cell: no image shift unless the atoms sit at
                     * opposite faces of a thin box, which g >= 3 rules out */
                    classify_shifted(pos + 3 * i, pos + 3 * j, zero, lo2, hi2, dmin2, i > j ? i : j,
                                     close_mark, band_mark);
                }
            for (int o = 0; o < 13; ++o) {
                int64_t u[3] = {cx + off[o][0], cy + off[o][1], cz + off[o][2]};
                double sh[3];
                for (int d = 0; d < 3; ++d) {
                    sh[d] = 0.0;
                    if (u[d] < 0) { u[d] += g[d]; sh[d] = -L[d]; }
                    else if (u[d] >= g[d]) { u[d] -= g[d]; sh[d] = L[d]; }
                }
                int64_t e = u[0] + g[0] * (u[1] + g[1] * u[2]);
                for (int64_t a = head[c]; a < head[c + 1]; ++a)
                    for (int64_t b = head[e]; b < head[e + 1]; ++b) {
                        int64_t i = order[a], j = order[b];
                        classify_shifted(pos + 3 * i, pos + 3 * j, sh, lo2, hi2, dmin2, i > j ? i : j,
                                         close_mark, band_mark);
                    }
            }
        }
        free(order);
        free(gid);
        free(head);
    }
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i) m += (close_mark[i] | band_mark[i]);
    return m;
}
