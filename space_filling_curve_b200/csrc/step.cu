// step.cu -- the per-step kernels: the skin check (a conservative skin keeps
// the neighbor graph valid between rebuilds; Tessera, abstract) and the fused
// edge-geometry + one-hop aggregation that each message-passing layer
// consumes (review of arXiv 2505.06711, "load-bearing attack" paragraph:
// each layer aggregates one-hop neighbor features within the cutoff).
#include "common.cuh"

#include <initializer_list>
#include <type_traits>

namespace tess {

// ---------------------------------------------------------------- skin check

__device__ __forceinline__ double min_image_d(double d, double L) {
    if (d > 0.5 * L) return d - L;
    if (d < -0.5 * L) return d + L;
    return d;
}

// max_i |minimg(r_i - r_i^ref)|^2 in fp64 (exact differences of fp32 values,
// one IEEE rounding per product and sum, no contraction), flag if > h2.
__global__ __launch_bounds__(256) void skin_kernel(const float4* __restrict__ pos, const float4* __restrict__ ref,
                                                   int n, double3 L, double h2, int32_t* __restrict__ rebuild,
                                                   unsigned long long* __restrict__ max_bits) {
    double m = 0.0;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float4 a = pos[i], b = ref[i];
        const double dx = min_image_d((double)a.x - (double)b.x, L.x);
        const double dy = min_image_d((double)a.y - (double)b.y, L.y);
        const double dz = min_image_d((double)a.z - (double)b.z, L.z);
        const double d2 = __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
        m = fmax(m, d2);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmax(m, __shfl_xor_sync(FULL, m, o));
    __shared__ double s[8];
    if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, s[w]);
        if (m > h2) atomicOr(rebuild, 1);
        // non-negative doubles order like their bit patterns
        if (max_bits) atomicMax(max_bits, (unsigned long long)__double_as_longlong(m));
    }
}

tess_status skin_check(const float* pos, const float* pos_ref, int n, tess_box box, float skin, int32_t* rebuild,
                       double* max_disp2, cudaStream_t s) {
    if (n <= 0 || !pos || !pos_ref || !rebuild || !(skin >= 0.f) || !std::isfinite(skin)) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (!aligned(pos, 16) || !aligned(pos_ref, 16) || (max_disp2 && !aligned(max_disp2, 8)))
        return TESS_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const double h = 0.5 * (double)skin;
    const double h2 = h * h;
    StageScope sc(ST_SKIN, s);
    cudaMemsetAsync(rebuild, 0, sizeof(int32_t), s);
    if (max_disp2) cudaMemsetAsync(max_disp2, 0, sizeof(double), s);
    const int blocks = (int)std::min<long long>(((long long)n + 255) / 256, (long long)sms * 8);
    skin_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(pos), reinterpret_cast<const float4*>(pos_ref),
                                       n, make_double3(box.lx, box.ly, box.lz), h2, rebuild,
                                       reinterpret_cast<unsigned long long*>(max_disp2));
    count_launch();
    return launch_status();
}

// ---------------------------------------------------------------- edge aggregate

struct EdgeArgs {
    const float4* pos;
    const int* nbr;
    const int* counts;
    const float* feat;
    float* out;
    float4* edge_vec;
    float* edge_fc;
    float4* edge_unit;
    int n, cap, F;
    float3 L;
    float rc, inv_rc2;
};

__device__ __forceinline__ float min_image_f(float d, float L) {
    if (d > 0.5f * L) return d - L;
    if (d < -0.5f * L) return d + L;
    return d;
}

// Smooth cosine cutoff f_c = (cos(pi r / rc) + 1) / 2 for r < rc, written
// in w = 1 - (r / rc)^2 in (0, 1]: f_c = cos^2(pi sqrt(1 - w) / 2) is an
// entire function of w whose Taylor series at w = 0 is w^2 (b_2 + b_3 w +
// ...).  Its coefficients follow from cos(pi sqrt(u)) = sum_k c_k u^k, c_k =
// (-pi^2)^k / (2k)!, by putting u = 1 - w: b_j = (-1)^j / 2 sum_{k >= j} c_k
// C(k, j) (b_0 = b_1 = 0, b_2 = pi^2 / 16).  Every b_j is positive, so the
// fp32 Horner sum has no cancellation and stays within ~2e-7 relative error
// on the whole range -- also next to the cutoff, where f_c ~ (pi^2/16) w^2
// vanishes.  Eight terms (b_2 .. b_9): truncation below 2e-9.  w itself is
// one fused multiply-add, 1 - r^2 / rc^2; no square root or trigonometric
// call is needed on the aggregation path.
__host__ __device__ constexpr double fc_w_coef(int j) {
    double s = 0.0;
    double c = 1.0;                  // c_k
    for (int k = 0; k <= 40; ++k) {
        if (k > 0) c *= -9.8696044010893586188 / ((2.0 * k - 1.0) * (2.0 * k));
        if (k >= j) {
            double bn = 1.0;         // C(k, j)
            for (int t = 1; t <= j; ++t) bn = bn * (double)(k - j + t) / (double)t;
            s += c * bn;
        }
    }
    return ((j & 1) ? -s : s) * 0.5;
}

__device__ __forceinline__ float cutoff_w(float w) {
    float q = (float)fc_w_coef(9);
    q = fmaf(q, w, (float)fc_w_coef(8));
    q = fmaf(q, w, (float)fc_w_coef(7));
    q = fmaf(q, w, (float)fc_w_coef(6));
    q = fmaf(q, w, (float)fc_w_coef(5));
    q = fmaf(q, w, (float)fc_w_coef(4));
    q = fmaf(q, w, (float)fc_w_coef(3));
    q = fmaf(q, w, (float)fc_w_coef(2));
    return (w * w) * q;
}

// d f_c / d w = w (2 b_2 + 3 b_3 w + ...), also all positive terms; then
// (d f_c / d r) / r = -(2 / rc^2) d f_c / d w.
__device__ __forceinline__ float cutoff_dw(float w) {
    float q = (float)(9.0 * fc_w_coef(9));
    q = fmaf(q, w, (float)(8.0 * fc_w_coef(8)));
    q = fmaf(q, w, (float)(7.0 * fc_w_coef(7)));
    q = fmaf(q, w, (float)(6.0 * fc_w_coef(6)));
    q = fmaf(q, w, (float)(5.0 * fc_w_coef(5)));
    q = fmaf(q, w, (float)(4.0 * fc_w_coef(4)));
    q = fmaf(q, w, (float)(3.0 * fc_w_coef(3)));
    q = fmaf(q, w, (float)(2.0 * fc_w_coef(2)));
    return w * q;
}

constexpr int EDGE_WARPS = 8;

// One warp per row i.  Lanes first compute the geometry of up to 32 edges
// at once (one edge per lane), then walk the accepted edges with the
// (j, f_c) pair broadcast and accumulate f_c * h_j over the feature
// dimension, VEC features per lane per step.
template <int VEC>
__global__ __launch_bounds__(EDGE_WARPS * 32) void edge_kernel(EdgeArgs A) {
    const int lane = threadIdx.x & 31;
    const long long row0 = (long long)blockIdx.x * EDGE_WARPS + (threadIdx.x >> 5);
    const long long rstride = (long long)gridDim.x * EDGE_WARPS;
    const bool edges = A.edge_vec || A.edge_fc || A.edge_unit;
    const int nfchunks = (A.F + 32 * VEC - 1) / (32 * VEC);
    for (long long i = row0; i < A.n; i += rstride) {
        const float4 pi = A.pos[i];
        const int m = min(A.counts[i], A.cap);
        const int limit = edges ? A.cap : max(m, 0);
        for (int fc0 = 0; fc0 < nfchunks; ++fc0) {
            float acc[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
            const int f0 = fc0 * 32 * VEC + lane * VEC;
            for (int b = 0; b < limit; b += 32) {
                const int s = b + lane;
                const size_t e = (size_t)i * A.cap + s;
                int j = -1;
                float fc = 0.f;
                if (s < m) j = A.nbr[e];
                if (j >= 0 && j < A.n) {
                    const float4 pj = A.pos[j];
                    const float dx = min_image_f(pj.x - pi.x, A.L.x);
                    const float dy = min_image_f(pj.y - pi.y, A.L.y);
                    const float dz = min_image_f(pj.z - pi.z, A.L.z);
                    const float r2 = fmaf(dz, dz, fmaf(dy, dy, dx * dx));
                    const float w = fmaf(-r2, A.inv_rc2, 1.0f);
                    fc = w > 0.0f ? cutoff_w(w) : 0.0f;
                    if (fc0 == 0 && edges) {
                        const float r = sqrtf(r2);
                        const float inv_r = r > 0.f ? 1.0f / r : 0.f;
                        if (A.edge_vec) A.edge_vec[e] = make_float4(dx, dy, dz, r);
                        if (A.edge_fc) A.edge_fc[e] = fc;
                        if (A.edge_unit) A.edge_unit[e] = make_float4(dx * inv_r, dy * inv_r, dz * inv_r, 0.f);
                    }
                } else {
                    j = -1;
                    if (fc0 == 0 && edges && s < A.cap) {
                        if (A.edge_vec) A.edge_vec[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (A.edge_fc) A.edge_fc[e] = 0.f;
                        if (A.edge_unit) A.edge_unit[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
                unsigned live = __ballot_sync(FULL, fc != 0.f);
                while (live) {
                    const int l = __ffs(live) - 1;
                    live &= live - 1;
                    const int jj = __shfl_sync(FULL, j, l);
                    const float w = __shfl_sync(FULL, fc, l);
                    const float* h = A.feat + (size_t)jj * A.F + f0;
                    if (VEC == 2 && f0 + 1 < A.F) {
                        const float2 hv = *reinterpret_cast<const float2*>(h);
                        acc[0] = fmaf(w, hv.x, acc[0]);
                        if (VEC > 1) acc[VEC - 1] = fmaf(w, hv.y, acc[VEC - 1]);
                    } else {
#pragma unroll
                        for (int v = 0; v < VEC; ++v)
                            if (f0 + v < A.F) acc[v] = fmaf(w, h[v], acc[v]);
                    }
                }
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v)
                if (f0 + v < A.F) A.out[(size_t)i * A.F + f0 + v] = acc[v];
        }
    }
}

#ifndef TESS_EV_WARPS
#define TESS_EV_WARPS 24
#endif
#ifndef TESS_EV_GEO_UNROLL
#define TESS_EV_GEO_UNROLL 4
#endif
#ifndef TESS_EV_ACC_UNROLL
#define TESS_EV_ACC_UNROLL 4
#endif
constexpr int EV_WARPS = TESS_EV_WARPS;
constexpr int EV_MAXCAP = 512;       // live edges of one row staged in shared memory
#ifndef TESS_EV_MINB
#define TESS_EV_MINB 1               // resident blocks per SM the register budget aims at
#endif
#ifndef TESS_EV_CHUNK
#define TESS_EV_CHUNK 768
#endif
#ifndef TESS_EV_W
#define TESS_EV_W 4                  // floats per feature load when F allows (4 or 8)
#endif
// Rows are taken in chunks of consecutive rows per block (chunks dealt to
// blocks round robin), so that the neighbor feature rows one row pulls into
// L1 serve the next rows too: rows adjacent in the sorted order are adjacent
// in space and share most of their neighbors.  All blocks together sweep a
// front of gridDim * chunk rows, which bounds the L2 working set.
constexpr int EV_CHUNK = TESS_EV_CHUNK;

// the shape for dense rows: caps above EV_DENSE_CAP (the row capacity stands
// in for the mean row length, which the host does not know)
constexpr int EV_DENSE_CAP = 192;
constexpr int EV_DENSE_WARPS = 8;
constexpr int EV_DENSE_MINB = 3;
constexpr int EV_DENSE_CHUNK = 256;
constexpr int EV_GEO_UNROLL = TESS_EV_GEO_UNROLL;     // neighbor/position loads in flight per lane
constexpr int EV_ACC_UNROLL = TESS_EV_ACC_UNROLL;     // feature rows in flight per lane group

// W consecutive floats of a feature row, held as W/2 packed pairs so that
// sm_100's paired fp32 instructions (fma.rn.f32x2, add.rn.f32x2) work on two
// features at once.  W = 4: one 16-byte load; W = 8: one 32-byte load, which
// sm_100 issues as a single instruction.
__device__ __forceinline__ unsigned long long f2_dup(float v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float f2_sum(unsigned long long a) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a));
    return lo + hi;
}
__device__ __forceinline__ unsigned long long f2_shfl_xor(unsigned long long a, int o) {
    unsigned lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(a));
    lo = __shfl_xor_sync(FULL, lo, o);
    hi = __shfl_xor_sync(FULL, hi, o);
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

template <int W>
struct FVec {
    unsigned long long p[W / 2];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int k = 0; k < W / 2; ++k) p[k] = 0ull;
    }
    // this += w * h, two features per instruction
    __device__ __forceinline__ void fma(float w, const FVec& h) {
        const unsigned long long w2 = f2_dup(w);
#pragma unroll
        for (int k = 0; k < W / 2; ++k) p[k] = f2_fma(w2, h.p[k], p[k]);
    }
    // acc2 + the products a_k b_k, summed pairwise into a packed pair
    __device__ __forceinline__ static unsigned long long dot2(const FVec& a, const FVec& b, unsigned long long acc2) {
#pragma unroll
        for (int k = 0; k < W / 2; ++k) acc2 = f2_fma(a.p[k], b.p[k], acc2);
        return acc2;
    }
    __device__ __forceinline__ void shfl_add(int o) {
#pragma unroll
        for (int k = 0; k < W / 2; ++k) p[k] = f2_add(p[k], f2_shfl_xor(p[k], o));
    }
    __device__ __forceinline__ void store(float* ptr) const {
        if (W == 4) {
            asm volatile("st.global.v2.b64 [%0], {%1, %2};" ::"l"(ptr), "l"(p[0]), "l"(p[1]) : "memory");
        } else {
            asm volatile("st.global.v2.b64 [%0], {%1, %2};" ::"l"(ptr), "l"(p[0]), "l"(p[1]) : "memory");
            asm volatile("st.global.v2.b64 [%0], {%1, %2};" ::"l"(ptr + 4), "l"(p[W / 2 - 2]), "l"(p[W / 2 - 1])
                         : "memory");
        }
    }
};

template <int W>
__device__ __forceinline__ FVec<W> ld_vec(const float* p);

template <>
__device__ __forceinline__ FVec<4> ld_vec<4>(const float* p) {
    FVec<4> r;
    asm("ld.global.v2.b64 {%0, %1}, [%2];" : "=l"(r.p[0]), "=l"(r.p[1]) : "l"(p));
    return r;
}

// 32-byte load (p 32-byte aligned); the features are read-only for the
// kernel's duration, so the load has no ordering constraint.
template <>
__device__ __forceinline__ FVec<8> ld_vec<8>(const float* p) {
    FVec<8> r;
    asm("ld.global.v4.b64 {%0, %1, %2, %3}, [%4];" : "=l"(r.p[0]), "=l"(r.p[1]), "=l"(r.p[2]), "=l"(r.p[3]) : "l"(p));
    return r;
}

// Features in vectors of W floats (F = W * LPE * VPL, F <= 256): LPE lanes
// share one edge and lane fl owns vectors v * LPE + fl (v < VPL) of the row,
// so one load instruction of a lane group reads LPE * W * 4 contiguous bytes
// (whole sectors) and a warp reads 32/LPE neighbor feature rows per step.
// Phase 1 computes the geometry of the whole row (one edge per lane, several
// loads in flight) and compacts the live (j, f_c) pairs into shared memory;
// phase 2 accumulates f_c * h_j with several rows in flight; the lane groups
// are then summed with shuffles.  Shared memory: EV_WARPS * cap int2
// (dynamic, so that what a small cap leaves over serves as L1).
// Block shape (WARPS per block, MINB resident blocks, rows per CHUNK): one
// block of 24 warps per SM over 768-row chunks for rows of up to ~100 live
// edges; dense rows (caps above 192) fill L1 faster and run best as 3 blocks
// of 8 warps over 256-row chunks.
template <int W, int LPE, int VPL, int WARPS = EV_WARPS, int MINB = TESS_EV_MINB, int CHUNK = EV_CHUNK>
__global__ __launch_bounds__(WARPS * 32, MINB) void edge_vec_kernel(EdgeArgs A) {
    constexpr int EPI = 32 / LPE;
    extern __shared__ int2 s_edge[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2* live_e = s_edge + (size_t)warp * A.cap;
    const int g = lane / LPE, fl = lane % LPE;
    const bool edges = A.edge_vec || A.edge_fc || A.edge_unit;
    for (long long c0 = (long long)blockIdx.x * CHUNK; c0 < A.n; c0 += (long long)gridDim.x * CHUNK)
    for (long long i = c0 + warp, c1 = min((long long)A.n, c0 + CHUNK); i < c1; i += WARPS) {
        const float4 pi = A.pos[i];
        const int m = max(min(A.counts[i], A.cap), 0);
        const int limit = edges ? A.cap : m;
        int nlive = 0;
        for (int s0 = 0; s0 < limit; s0 += 32 * EV_GEO_UNROLL) {
            int j[EV_GEO_UNROLL];
            float4 pj[EV_GEO_UNROLL];
#pragma unroll
            for (int u = 0; u < EV_GEO_UNROLL; ++u) {
                const int s = s0 + u * 32 + lane;
                j[u] = (s < m) ? A.nbr[(size_t)i * A.cap + s] : -1;
                if (j[u] >= A.n) j[u] = -1;
            }
#pragma unroll
            for (int u = 0; u < EV_GEO_UNROLL; ++u)
                if (j[u] >= 0) pj[u] = A.pos[j[u]];
#pragma unroll
            for (int u = 0; u < EV_GEO_UNROLL; ++u) {
                const int s = s0 + u * 32 + lane;
                float fc = 0.f;
                if (j[u] >= 0) {
                    const float dx = min_image_f(pj[u].x - pi.x, A.L.x);
                    const float dy = min_image_f(pj[u].y - pi.y, A.L.y);
                    const float dz = min_image_f(pj[u].z - pi.z, A.L.z);
                    const float r2 = fmaf(dz, dz, fmaf(dy, dy, dx * dx));
                    const float w = fmaf(-r2, A.inv_rc2, 1.0f);
                    fc = w > 0.0f ? cutoff_w(w) : 0.0f;
                    if (edges) {
                        const size_t e = (size_t)i * A.cap + s;
                        const float r = sqrtf(r2);
                        const float inv_r = r > 0.f ? 1.0f / r : 0.f;
                        if (A.edge_vec) A.edge_vec[e] = make_float4(dx, dy, dz, r);
                        if (A.edge_fc) A.edge_fc[e] = fc;
                        if (A.edge_unit) A.edge_unit[e] = make_float4(dx * inv_r, dy * inv_r, dz * inv_r, 0.f);
                    }
                } else if (edges && s < A.cap) {
                    const size_t e = (size_t)i * A.cap + s;
                    if (A.edge_vec) A.edge_vec[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (A.edge_fc) A.edge_fc[e] = 0.f;
                    if (A.edge_unit) A.edge_unit[e] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                const unsigned live = __ballot_sync(FULL, fc != 0.f);
                if (fc != 0.f) live_e[nlive + __popc(live & lanemask_lt())] = make_int2(j[u], __float_as_int(fc));
                nlive += __popc(live);
            }
        }
        __syncwarp();
        FVec<W> acc[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc[v].zero();
        const float* fbase = A.feat + fl * W;
        for (int e0 = 0; e0 < nlive; e0 += EPI * EV_ACC_UNROLL) {
            int2 ed[EV_ACC_UNROLL];
            FVec<W> h[EV_ACC_UNROLL][VPL];
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                const int e = e0 + u * EPI + g;
                ed[u] = (e < nlive) ? live_e[e] : make_int2(-1, 0);
            }
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                const float* src = fbase + (size_t)max(ed[u].x, 0) * A.F;
#pragma unroll
                for (int v = 0; v < VPL; ++v) h[u][v] = ld_vec<W>(src + v * LPE * W);
            }
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                if (ed[u].x < 0) continue;     // past the last live edge
                const float w = __int_as_float(ed[u].y);
#pragma unroll
                for (int v = 0; v < VPL; ++v) acc[v].fma(w, h[u][v]);
            }
        }
#pragma unroll
        for (int o = LPE; o < 32; o <<= 1) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) acc[v].shfl_add(o);
        }
        if (g == 0) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) acc[v].store(A.out + (size_t)i * A.F + (v * LPE + fl) * W);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------- backward (force path)

struct BackArgs {
    const float4* pos;
    const int* nbr;
    const int* counts;
    const float* feat;
    const float* grad_out;
    float* grad_feat;
    float* grad_pos;
    int n, cap, F;
    float3 L;
    float inv_rc2;
    float dfc_scale;     // -2 / rc^2: (d f_c / d r) / r = dfc_scale * cutoff_dw(w)
};

// Vector-Jacobian product of the aggregation over a full symmetric list
// (j in row i exactly when i in row j, as tess_build_neighbors writes it):
//   grad_feat[i] = sum_{j in row i} f_c(r_ij) g_j
//   grad_pos[i]  = -sum_{j in row i} f_c'(r_ij) (g_i . h_j + g_j . h_i) r_ij / |r_ij|
// The symmetry turns the scatter of the chain rule into a per-row gather, so
// no atomics.  Same layout as edge_vec_kernel: phase 1 geometry and live-edge
// compaction, phase 2 LPE lanes per edge with VPL vectors of h_j and g_j
// each.  Each lane keeps its own share of the force, sum over edges of (its
// part of the dot product) times (f_c'/r) r_ij, which is linear in the parts,
// so the lanes are summed once per row instead of once per edge.
#ifndef TESS_BK_WARPS
#define TESS_BK_WARPS 8
#endif
constexpr int BK_WARPS = TESS_BK_WARPS;
constexpr int BK_MAXCAP = 512;
#ifndef TESS_BK_CHUNK
#define TESS_BK_CHUNK 512
#endif
#ifndef TESS_BK_MINB
#define TESS_BK_MINB 3
#endif
constexpr int BK_CHUNK = TESS_BK_CHUNK;
#ifndef TESS_BK_ACC_UNROLL
#define TESS_BK_ACC_UNROLL 2
#endif
constexpr int BK_ACC_UNROLL = TESS_BK_ACC_UNROLL;   // edge steps in flight per lane group
#ifndef TESS_BK_PREFETCH
#define TESS_BK_PREFETCH 1
#endif

template <int W, int LPE, int VPL>
__global__ __launch_bounds__(BK_WARPS * 32, TESS_BK_MINB) void edge_backward_kernel(BackArgs A) {
    constexpr int EPI = 32 / LPE;
    // dynamic: BK_WARPS * cap float4 (f_c, v.x, v.y, v.z) with v = (f_c'/r) r_ij,
    // then BK_WARPS * cap int (j)
    extern __shared__ float4 s_dyn[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float4* s_w = s_dyn + (size_t)warp * A.cap;
    int* s_j = reinterpret_cast<int*>(s_dyn + (size_t)BK_WARPS * A.cap) + (size_t)warp * A.cap;
    const int g = lane / LPE, fl = lane % LPE;
    for (long long c0 = (long long)blockIdx.x * BK_CHUNK; c0 < A.n; c0 += (long long)gridDim.x * BK_CHUNK)
    for (long long i = c0 + warp, c1 = min((long long)A.n, c0 + BK_CHUNK); i < c1; i += BK_WARPS) {
        const float4 pi = A.pos[i];
        const int m = max(min(A.counts[i], A.cap), 0);
        int nlive = 0;
        for (int s0 = 0; s0 < m; s0 += 32) {
            const int s = s0 + lane;
            int j = (s < m) ? A.nbr[(size_t)i * A.cap + s] : -1;
            if (j >= A.n) j = -1;
            float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
            bool live = false;
            if (j >= 0) {
                const float4 pj = A.pos[j];
                const float dx = min_image_f(pj.x - pi.x, A.L.x);
                const float dy = min_image_f(pj.y - pi.y, A.L.y);
                const float dz = min_image_f(pj.z - pi.z, A.L.z);
                const float ww = fmaf(-fmaf(dz, dz, fmaf(dy, dy, dx * dx)), A.inv_rc2, 1.0f);
                if (ww > 0.0f) {
                    const float dr = A.dfc_scale * cutoff_dw(ww);
                    w = make_float4(cutoff_w(ww), dr * dx, dr * dy, dr * dz);
                    live = true;
                }
            }
            const unsigned bm = __ballot_sync(FULL, live);
            if (live) {
                const int k = nlive + __popc(bm & lanemask_lt());
                s_j[k] = j;
                s_w[k] = w;
            }
            nlive += __popc(bm);
        }
        __syncwarp();
        const size_t own = (size_t)i * A.F + fl * W;
        FVec<W> gi[VPL], hi[VPL], acc[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            gi[v] = ld_vec<W>(A.grad_out + own + v * LPE * W);
            hi[v] = ld_vec<W>(A.feat + own + v * LPE * W);
            acc[v].zero();
        }
#if TESS_BK_PREFETCH
        {
            // the next row of this warp: its list entries into L2 meanwhile
            long long in = i + BK_WARPS;
            if (in >= c1) in = c0 + (long long)gridDim.x * BK_CHUNK + warp;
            if (in < A.n && lane * 32 < A.cap)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(A.nbr + (size_t)in * A.cap + lane * 32));
        }
#endif
        float fx = 0.f, fy = 0.f, fz = 0.f;
        // BK_ACC_UNROLL steps of EPI edges in flight per lane group
        for (int e0 = 0; e0 < nlive; e0 += EPI * BK_ACC_UNROLL) {
            int jj[BK_ACC_UNROLL];
            float4 ww[BK_ACC_UNROLL];
#pragma unroll
            for (int u = 0; u < BK_ACC_UNROLL; ++u) {
                const int e = e0 + u * EPI + g;
                const bool ok = e < nlive;
                jj[u] = ok ? s_j[e] : -1;
                ww[u] = ok ? s_w[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            FVec<W> hj[BK_ACC_UNROLL][VPL], gj[BK_ACC_UNROLL][VPL];
#pragma unroll
            for (int u = 0; u < BK_ACC_UNROLL; ++u) {
                const size_t base = (size_t)(jj[u] >= 0 ? jj[u] : (int)i) * A.F + fl * W;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    hj[u][v] = ld_vec<W>(A.feat + base + v * LPE * W);
                    gj[u][v] = ld_vec<W>(A.grad_out + base + v * LPE * W);
                }
            }
#pragma unroll
            for (int u = 0; u < BK_ACC_UNROLL; ++u) {
                if (jj[u] < 0) continue;
                unsigned long long d2 = 0ull;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    acc[v].fma(ww[u].x, gj[u][v]);
                    d2 = FVec<W>::dot2(gi[v], hj[u][v], d2);
                    d2 = FVec<W>::dot2(gj[u][v], hi[v], d2);
                }
                const float dot = f2_sum(d2);
                fx = fmaf(dot, ww[u].y, fx);
                fy = fmaf(dot, ww[u].z, fy);
                fz = fmaf(dot, ww[u].w, fz);
            }
        }
        // feature gradient: lane groups hold disjoint edges of the same
        // features; force: every lane holds a share
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            fx += __shfl_xor_sync(FULL, fx, o);
            fy += __shfl_xor_sync(FULL, fy, o);
            fz += __shfl_xor_sync(FULL, fz, o);
        }
#pragma unroll
        for (int o = LPE; o < 32; o <<= 1) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) acc[v].shfl_add(o);
        }
        if (g == 0) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) acc[v].store(A.grad_feat + own + v * LPE * W);
        }
        if (lane == 0) {
            A.grad_pos[3 * (size_t)i] = -fx;
            A.grad_pos[3 * (size_t)i + 1] = -fy;
            A.grad_pos[3 * (size_t)i + 2] = -fz;
        }
        __syncwarp();
    }
}

// Grid of a chunked row walk for `kernel` (`threads` per block, `smem`
// dynamic bytes, `chunk` rows per chunk): CHUNK_WAVES times the blocks that
// are resident at once, never more blocks than chunks.  With a single
// resident wave the slowest block sets the kernel time and its time varies
// from launch to launch (measured at 10.24M atoms, 40 launches: aggregation
// median 15.7 ms, max 16.9); with four waves the hardware scheduler starts a
// new block wherever one finishes (median 13.7 ms, max 14.2).  Blocks per SM come from the kernel's registers and
// thread count alone; the shared-memory carveout is then set to the smallest
// configuration that holds that many blocks, so that the rest of the SM's
// 256 KB serves as L1 for the gathers (the driver may otherwise keep a
// larger carveout than the launch needs).  Deriving the block count from the
// carveout instead would feed back: a carveout rounded down lowers the
// count, which lowers the next carveout.
constexpr int CHUNK_WAVES = 4;

template <class K>
int chunk_grid(K* kernel, int threads, size_t smem, int n, int sms, int chunk) {
    static const int configs_kb[] = {0, 8, 16, 32, 64, 100, 132, 164, 196, 228};
    int dev = 0, max_sm = 0, regs_sm = 65536, thr_sm = 2048;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&max_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
    cudaFuncAttributes fa{};
    int per_sm = 1;
    if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess && fa.numRegs > 0) {
        const int regs_block = ((fa.numRegs * 32 + 255) / 256 * 256) * (threads / 32);    // per-warp allocation unit
        per_sm = std::max(1, std::min(regs_sm / regs_block, thr_sm / threads));
    }
    if (max_sm > 0) {
        const size_t need = (size_t)per_sm * (smem + fa.sharedSizeBytes + 1024);
        int kb = configs_kb[sizeof(configs_kb) / sizeof(int) - 1];
        for (int c : configs_kb)
            if ((size_t)c * 1024 >= need) {
                kb = c;
                break;
            }
        const int pct = std::min(100, (kb * 1024 * 100 + max_sm - 1) / max_sm);
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) == cudaSuccess && occ > 0)
        per_sm = std::min(per_sm, occ);
    const long long chunks = ((long long)n + chunk - 1) / chunk;
    return (int)std::max<long long>(1, std::min<long long>(chunks, (long long)sms * per_sm * CHUNK_WAVES));
}

template <int V>
using ic = std::integral_constant<int, V>;

// Launch shape for q = F / W vectors per row (q a power of two): calls
// launch(W, LPE, VPL) as integral constants; false when q is not covered.
template <int W, class Launch>
bool by_shape(int q, Launch&& launch) {
    if (W == 4) {
        switch (q) {
            case 1: launch(ic<W>{}, ic<1>{}, ic<1>{}); return true;
            case 2: launch(ic<W>{}, ic<2>{}, ic<1>{}); return true;
            case 4: launch(ic<W>{}, ic<2>{}, ic<2>{}); return true;
            case 8: launch(ic<W>{}, ic<4>{}, ic<2>{}); return true;
            case 16: launch(ic<W>{}, ic<8>{}, ic<2>{}); return true;
            case 32: launch(ic<W>{}, ic<16>{}, ic<2>{}); return true;
            case 64: launch(ic<W>{}, ic<32>{}, ic<2>{}); return true;
            default: return false;
        }
    }
    switch (q) {
        case 1: launch(ic<W>{}, ic<1>{}, ic<1>{}); return true;
        case 2: launch(ic<W>{}, ic<2>{}, ic<1>{}); return true;
        case 4: launch(ic<W>{}, ic<4>{}, ic<1>{}); return true;
        case 8: launch(ic<W>{}, ic<8>{}, ic<1>{}); return true;
        case 16: launch(ic<W>{}, ic<8>{}, ic<2>{}); return true;
        case 32: launch(ic<W>{}, ic<16>{}, ic<2>{}); return true;
        default: return false;
    }
}

// Vector width for feature rows of F floats whose arrays are `ptrs`: 8 when
// F is a multiple of 8 and every array is 32-byte aligned, else 4 (the
// callers require 16-byte alignment and F % 4 == 0 for either).
inline int pick_width(int F, std::initializer_list<const void*> ptrs) {
    bool wide = TESS_EV_W == 8 && F % 8 == 0;
    for (const void* p : ptrs) wide = wide && aligned(p, 32);
    return wide ? 8 : 4;
}

tess_status edge_backward(const float* pos, int n, tess_box box, float rc, const int32_t* nbr, const int32_t* counts,
                          int cap, const float* feat, const float* grad_out, int F, float* grad_feat,
                          float* grad_pos, cudaStream_t s) {
    if (n <= 0 || !pos || !nbr || !counts || !feat || !grad_out || !grad_feat || !grad_pos || cap < 1 || F < 1)
        return TESS_ERR_INVALID_ARG;
    if (!(rc > 0.f) || !std::isfinite(rc)) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (F % 4 != 0 || F > 256 || cap > BK_MAXCAP || !aligned(pos, 16) || !aligned(feat, 16) ||
        !aligned(grad_out, 16) || !aligned(grad_feat, 16))
        return TESS_ERR_INVALID_ARG;
    if (box.lx < 2.f * rc || box.ly < 2.f * rc || box.lz < 2.f * rc) return TESS_ERR_BOX_TOO_SMALL;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    BackArgs A;
    A.pos = reinterpret_cast<const float4*>(pos);
    A.nbr = nbr;
    A.counts = counts;
    A.feat = feat;
    A.grad_out = grad_out;
    A.grad_feat = grad_feat;
    A.grad_pos = grad_pos;
    A.n = n;
    A.cap = cap;
    A.F = F;
    A.L = make_float3(box.lx, box.ly, box.lz);
    A.inv_rc2 = 1.0f / (rc * rc);
    A.dfc_scale = (float)(-2.0 / ((double)rc * (double)rc));
    StageScope sc(ST_BACKWARD, s);
    const size_t smem = (size_t)BK_WARPS * cap * (sizeof(float4) + sizeof(int));
    auto launch = [&](auto w, auto lpe, auto vpl) {
        auto* k = edge_backward_kernel<decltype(w)::value, decltype(lpe)::value, decltype(vpl)::value>;
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<chunk_grid(k, BK_WARPS * 32, smem, n, sms, BK_CHUNK), BK_WARPS * 32, smem, s>>>(A);
    };
    const int W = pick_width(F, {feat, grad_out, grad_feat});
    const bool ok = W == 8 ? by_shape<8>(F / 8, launch) : by_shape<4>(F / 4, launch);
    if (!ok) return TESS_ERR_INVALID_ARG;    // F a multiple of 4 that is not 4 * 2^k
    count_launch();
    return launch_status();
}

tess_status edge_aggregate(const float* pos, int n, tess_box box, float rc, const int32_t* nbr, const int32_t* counts,
                           int cap, const float* feat, int F, float* out, float* edge_vec, float* edge_fc,
                           float* edge_unit, cudaStream_t s) {
    if (n <= 0 || !pos || !nbr || !counts || !feat || !out || cap < 1 || F < 1) return TESS_ERR_INVALID_ARG;
    if (!(rc > 0.f) || !std::isfinite(rc)) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (!aligned(pos, 16) || (edge_vec && !aligned(edge_vec, 16)) || (edge_unit && !aligned(edge_unit, 16)))
        return TESS_ERR_INVALID_ARG;
    if (box.lx < 2.f * rc || box.ly < 2.f * rc || box.lz < 2.f * rc) return TESS_ERR_BOX_TOO_SMALL;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    EdgeArgs A;
    A.pos = reinterpret_cast<const float4*>(pos);
    A.nbr = nbr;
    A.counts = counts;
    A.feat = feat;
    A.out = out;
    A.edge_vec = reinterpret_cast<float4*>(edge_vec);
    A.edge_fc = edge_fc;
    A.edge_unit = reinterpret_cast<float4*>(edge_unit);
    A.n = n;
    A.cap = cap;
    A.F = F;
    A.L = make_float3(box.lx, box.ly, box.lz);
    A.rc = rc;
    A.inv_rc2 = 1.0f / (rc * rc);
    StageScope sc(ST_EDGE, s);
    const long long rows_blocks = ((long long)n + EDGE_WARPS - 1) / EDGE_WARPS;
    const int blocks = (int)std::min<long long>(rows_blocks, (long long)sms * 64);
    const bool vec = (F % 4 == 0) && F <= 256 && aligned(feat, 16) && aligned(out, 16) && cap <= EV_MAXCAP;
    const bool dense = cap > EV_DENSE_CAP;
    const int warps = dense ? EV_DENSE_WARPS : EV_WARPS;
    const size_t vsmem = (size_t)warps * cap * sizeof(int2);
    bool launched = false;
    if (vec) {
        auto launch = [&](auto w, auto lpe, auto vpl) {
            constexpr int Wv = decltype(w)::value, Lv = decltype(lpe)::value, Vv = decltype(vpl)::value;
            auto go = [&](auto* k, int chunk) {
                if (vsmem > 48 * 1024)
                    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)vsmem);
                k<<<chunk_grid(k, warps * 32, vsmem, n, sms, chunk), warps * 32, vsmem, s>>>(A);
            };
            if (dense) go(edge_vec_kernel<Wv, Lv, Vv, EV_DENSE_WARPS, EV_DENSE_MINB, EV_DENSE_CHUNK>, EV_DENSE_CHUNK);
            else go(edge_vec_kernel<Wv, Lv, Vv>, EV_CHUNK);
        };
        const int W = pick_width(F, {feat, out});
        launched = W == 8 ? by_shape<8>(F / 8, launch) : by_shape<4>(F / 4, launch);
    }
    if (!launched) {
        if ((F % 2 == 0) && aligned(feat, 8) && F >= 64) edge_kernel<2><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
        else edge_kernel<1><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
    }
    count_launch();
    return launch_status();
}

// ---------------------------------------------------------------- closest listed pair

// The closest pair the list holds -- a structural check for atoms that come
// anomalously close (Tessera runs are checked for such pairs; Tessera,
// abstract).  Squared distances as the skin check computes them: fp64 from
// the fp32 coordinates, one IEEE rounding per product and sum, no
// contraction.  Order: (r2, i, j) lexicographic, so ties go to the smallest
// pair.  One warp per row; per-block minima go to the workspace and one
// block reduces them.
constexpr int MP_THREADS = 256;
constexpr int MP_MAX_BLOCKS = 4096;

struct MinPairCand {
    unsigned long long r2;    // bits of the fp64 r2 (non-negative: ordered as integers)
    unsigned long long ij;    // (i << 32) | j
};

__device__ __forceinline__ bool mp_less(unsigned long long ar, unsigned long long aij, unsigned long long br,
                                        unsigned long long bij) {
    return ar < br || (ar == br && aij < bij);
}

__device__ __forceinline__ unsigned long long shfl_xor_u64s(unsigned long long v, int m) {
    const unsigned lo = __shfl_xor_sync(FULL, (unsigned)v, m);
    const unsigned hi = __shfl_xor_sync(FULL, (unsigned)(v >> 32), m);
    return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ void mp_warp_min(unsigned long long& r, unsigned long long& ij) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long orr = shfl_xor_u64s(r, o), oij = shfl_xor_u64s(ij, o);
        if (mp_less(orr, oij, r, ij)) {
            r = orr;
            ij = oij;
        }
    }
}

__global__ __launch_bounds__(MP_THREADS) void min_pair_kernel(const float4* __restrict__ pos, int n, double3 L,
                                                              const int* __restrict__ nbr,
                                                              const int* __restrict__ counts, int cap,
                                                              MinPairCand* __restrict__ cand) {
    __shared__ unsigned long long s_r[MP_THREADS / 32], s_ij[MP_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long br = ~0ull, bij = ~0ull;
    // chunks of consecutive rows per block, as in the aggregation: the rows'
    // neighbors overlap, so their positions stay in L1
    for (long long c0 = (long long)blockIdx.x * EV_CHUNK; c0 < n; c0 += (long long)gridDim.x * EV_CHUNK)
    for (long long i = c0 + warp, c1 = min((long long)n, c0 + EV_CHUNK); i < c1; i += MP_THREADS / 32) {
        const float4 pi = pos[i];
        const int m = max(min(counts[i], cap), 0);
        constexpr int U = 4;     // list entries in flight per lane
        for (int s0 = 0; s0 < m; s0 += 32 * U) {
            int j[U];
            float4 pj[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int s = s0 + 32 * u + lane;
                j[u] = s < m ? nbr[(size_t)i * cap + s] : -1;
                if (j[u] >= n) j[u] = -1;
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (j[u] >= 0) pj[u] = pos[j[u]];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (j[u] < 0) continue;
                const double dx = min_image_d((double)pj[u].x - (double)pi.x, L.x);
                const double dy = min_image_d((double)pj[u].y - (double)pi.y, L.y);
                const double dz = min_image_d((double)pj[u].z - (double)pi.z, L.z);
                const double r2 = __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
                const unsigned long long rb = (unsigned long long)__double_as_longlong(r2);
                const unsigned long long ij = ((unsigned long long)i << 32) | (unsigned)j[u];
                if (mp_less(rb, ij, br, bij)) {
                    br = rb;
                    bij = ij;
                }
            }
        }
    }
    mp_warp_min(br, bij);
    if (lane == 0) {
        s_r[warp] = br;
        s_ij[warp] = bij;
    }
    __syncthreads();
    if (warp == 0) {
        br = lane < MP_THREADS / 32 ? s_r[lane] : ~0ull;
        bij = lane < MP_THREADS / 32 ? s_ij[lane] : ~0ull;
        mp_warp_min(br, bij);
        if (lane == 0) cand[blockIdx.x] = MinPairCand{br, bij};
    }
}

__global__ __launch_bounds__(1024) void min_pair_reduce(const MinPairCand* __restrict__ cand, int nc,
                                                        double* __restrict__ r2_out, int32_t* __restrict__ pair_out) {
    __shared__ unsigned long long s_r[32], s_ij[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long br = ~0ull, bij = ~0ull;
    for (int k = threadIdx.x; k < nc; k += blockDim.x)
        if (mp_less(cand[k].r2, cand[k].ij, br, bij)) {
            br = cand[k].r2;
            bij = cand[k].ij;
        }
    mp_warp_min(br, bij);
    if (lane == 0) {
        s_r[warp] = br;
        s_ij[warp] = bij;
    }
    __syncthreads();
    if (warp == 0) {
        br = s_r[lane];
        bij = s_ij[lane];
        mp_warp_min(br, bij);
        if (lane == 0) {
            const bool none = bij == ~0ull;
            r2_out[0] = none ? __longlong_as_double(0x7ff0000000000000ll) : __longlong_as_double((long long)br);
            pair_out[0] = none ? -1 : (int32_t)(bij >> 32);
            pair_out[1] = none ? -1 : (int32_t)(unsigned)bij;
        }
    }
}

size_t min_pair_workspace() { return MP_MAX_BLOCKS * sizeof(MinPairCand); }

tess_status min_pair_distance(const float* pos, int n, tess_box box, const int32_t* nbr, const int32_t* counts,
                              int cap, void* ws, size_t ws_bytes, double* min_r2, int32_t* min_pair,
                              cudaStream_t s) {
    if (n <= 0 || !pos || !nbr || !counts || !ws || !min_r2 || !min_pair || cap < 1) return TESS_ERR_INVALID_ARG;
    if (!finite_pos(box.lx) || !finite_pos(box.ly) || !finite_pos(box.lz)) return TESS_ERR_INVALID_ARG;
    if (!aligned(pos, 16) || !aligned(ws, 16)) return TESS_ERR_INVALID_ARG;
    if (ws_bytes < min_pair_workspace()) return TESS_ERR_WORKSPACE_TOO_SMALL;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one resident wave (no more blocks than the workspace holds)
    const int blocks = std::min(chunk_grid(min_pair_kernel, MP_THREADS, 0, n, sms, EV_CHUNK), MP_MAX_BLOCKS);
    MinPairCand* cand = static_cast<MinPairCand*>(ws);
    StageScope sc(ST_MONITOR, s);
    min_pair_kernel<<<blocks, MP_THREADS, 0, s>>>(reinterpret_cast<const float4*>(pos), n,
                                                  make_double3(box.lx, box.ly, box.lz), nbr, counts, cap, cand);
    min_pair_reduce<<<1, 1024, 0, s>>>(cand, blocks, min_r2, min_pair);
    count_launch(2);
    return launch_status();
}

}  // namespace tess
