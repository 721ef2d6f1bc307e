// step.cu -- the per-step kernels: the skin check ("a conservative neighbor
// skin preserves topology across updates", Tessera, abstract) and the fused
// edge-geometry + one-hop aggregation that each message-passing layer
// consumes (review of arXiv 2505.06711, "load-bearing attack" paragraph:
// each layer aggregates one-hop neighbor features within the cutoff).
#include "common.cuh"

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

// Smooth cosine cutoff f_c = (cos(pi r / rc) + 1) / 2 for r < rc, as a
// function of u = (r / rc)^2 in [0, 1): cos(pi sqrt(u)) is the Taylor series
// sum_k (-pi^2 u)^k / (2k)!, which converges on the whole interval; eleven
// terms leave a truncation error below 4e-9 at u = 1 and the fp32 Horner
// evaluation adds a few 1e-7 at most (the largest partial terms are ~4).
// No square root or trigonometric call is needed on the aggregation path.
__host__ __device__ constexpr double cos_pi_sqrt_coef(int k) {
    double c = 1.0;
    for (int m = 1; m <= k; ++m) c *= -9.8696044010893586188 / ((2.0 * m - 1.0) * (2.0 * m));
    return c;
}

__device__ __forceinline__ float cutoff_u(float u) {
    float p = (float)cos_pi_sqrt_coef(10);
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(9));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(8));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(7));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(6));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(5));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(4));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(3));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(2));
    p = fmaf(p, u, (float)cos_pi_sqrt_coef(1));
    p = fmaf(p, u, 1.0f);
    return 0.5f * (p + 1.0f);
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
                    const float u = r2 * A.inv_rc2;
                    fc = u < 1.0f ? cutoff_u(u) : 0.0f;
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

constexpr int EV_WARPS = 8;
constexpr int EV_MAXCAP = 512;       // live edges of one row staged in shared memory
constexpr int EV_GEO_UNROLL = 4;     // neighbor/position loads in flight per lane
constexpr int EV_ACC_UNROLL = 4;     // feature rows in flight per lane group

// Features as float4 (F % 4 == 0, F <= 256): LPE lanes share one edge and
// each lane owns VPL float4 of the feature row (F = 4 * LPE * VPL), float4
// number v * LPE + fl for lane fl, so that one load instruction of a lane
// group reads LPE * 16 contiguous bytes (whole sectors, one cache line per
// edge at LPE = 8) and a warp reads 32/LPE neighbor feature rows per step.  Phase 1
// computes the geometry of the whole row (one edge per lane, several loads in
// flight) and compacts the live (j, f_c) pairs into shared memory; phase 2
// accumulates f_c * h_j with several rows in flight; the lane groups are then
// summed with shuffles.
template <int LPE, int VPL>
__global__ __launch_bounds__(EV_WARPS * 32, 3) void edge_vec4_kernel(EdgeArgs A) {
    constexpr int EPI = 32 / LPE;
    __shared__ int2 s_edge[EV_WARPS][EV_MAXCAP];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2* live_e = s_edge[warp];
    const int g = lane / LPE, fl = lane % LPE;
    const int F4 = A.F / 4;
    const float4* feat4 = reinterpret_cast<const float4*>(A.feat);
    float4* out4 = reinterpret_cast<float4*>(A.out);
    const bool edges = A.edge_vec || A.edge_fc || A.edge_unit;
    for (long long i = (long long)blockIdx.x * EV_WARPS + warp; i < A.n; i += (long long)gridDim.x * EV_WARPS) {
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
                    const float u2 = r2 * A.inv_rc2;
                    fc = u2 < 1.0f ? cutoff_u(u2) : 0.0f;
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
        float4 acc[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4* fbase = feat4 + fl;
        for (int e0 = 0; e0 < nlive; e0 += EPI * EV_ACC_UNROLL) {
            int2 ed[EV_ACC_UNROLL];
            float4 h[EV_ACC_UNROLL][VPL];
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                const int e = e0 + u * EPI + g;
                ed[u] = (e < nlive) ? live_e[e] : make_int2(-1, 0);
            }
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                const float4* src = fbase + (size_t)max(ed[u].x, 0) * F4;
#pragma unroll
                for (int v = 0; v < VPL; ++v) h[u][v] = src[v * LPE];
            }
#pragma unroll
            for (int u = 0; u < EV_ACC_UNROLL; ++u) {
                if (ed[u].x < 0) continue;     // past the last live edge
                const float w = __int_as_float(ed[u].y);
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    acc[v].x = fmaf(w, h[u][v].x, acc[v].x);
                    acc[v].y = fmaf(w, h[u][v].y, acc[v].y);
                    acc[v].z = fmaf(w, h[u][v].z, acc[v].z);
                    acc[v].w = fmaf(w, h[u][v].w, acc[v].w);
                }
            }
        }
#pragma unroll
        for (int o = LPE; o < 32; o <<= 1) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                acc[v].x += __shfl_xor_sync(FULL, acc[v].x, o);
                acc[v].y += __shfl_xor_sync(FULL, acc[v].y, o);
                acc[v].z += __shfl_xor_sync(FULL, acc[v].z, o);
                acc[v].w += __shfl_xor_sync(FULL, acc[v].w, o);
            }
        }
        if (g == 0) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) out4[(size_t)i * F4 + v * LPE + fl] = acc[v];
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------- backward (force path)

// sin(pi sqrt(u)) / (pi sqrt(u)) as the Taylor series sum_k (-pi^2 u)^k /
// (2k+1)!, eleven terms (truncation below 2e-10 at u = 1), so that
// d f_c / d r divided by r is -(pi^2 / (2 rc^2)) times this, with no root.
__host__ __device__ constexpr double sinc_pi_sqrt_coef(int k) {
    double c = 1.0;
    for (int m = 1; m <= k; ++m) c *= -9.8696044010893586188 / ((2.0 * m) * (2.0 * m + 1.0));
    return c;
}

__device__ __forceinline__ float sinc_u(float u) {
    float p = (float)sinc_pi_sqrt_coef(10);
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(9));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(8));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(7));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(6));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(5));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(4));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(3));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(2));
    p = fmaf(p, u, (float)sinc_pi_sqrt_coef(1));
    return fmaf(p, u, 1.0f);
}

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
    float dfc_scale;     // -(pi^2 / (2 rc^2)): (d f_c / d r) / r = dfc_scale * sinc_u(u)
};

// Vector-Jacobian product of the aggregation over a full symmetric list
// (j in row i exactly when i in row j, as tess_build_neighbors writes it):
//   grad_feat[i] = sum_{j in row i} f_c(r_ij) g_j
//   grad_pos[i]  = -sum_{j in row i} f_c'(r_ij) (g_i . h_j + g_j . h_i) r_ij / |r_ij|
// The symmetry turns the scatter of the chain rule into a per-row gather, so
// no atomics.  Same layout as edge_vec4_kernel: phase 1 geometry and live-edge
// compaction, phase 2 LPE lanes per edge with VPL float4 of h_j and g_j each;
// the edge's dot product is reduced within its lane group.
constexpr int BK_WARPS = 4;
constexpr int BK_MAXCAP = 512;

template <int LPE, int VPL>
__global__ __launch_bounds__(BK_WARPS * 32, 4) void edge_backward_kernel(BackArgs A) {
    constexpr int EPI = 32 / LPE;
    __shared__ int s_j[BK_WARPS][BK_MAXCAP];
    __shared__ float4 s_w[BK_WARPS][BK_MAXCAP];    // (f_c, v.x, v.y, v.z) with v = (f_c'/r) r_ij
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / LPE, fl = lane % LPE;
    const int F4 = A.F / 4;
    const float4* h4 = reinterpret_cast<const float4*>(A.feat);
    const float4* g4 = reinterpret_cast<const float4*>(A.grad_out);
    float4* gf4 = reinterpret_cast<float4*>(A.grad_feat);
    for (long long i = (long long)blockIdx.x * BK_WARPS + warp; i < A.n; i += (long long)gridDim.x * BK_WARPS) {
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
                const float u2 = fmaf(dz, dz, fmaf(dy, dy, dx * dx)) * A.inv_rc2;
                if (u2 < 1.0f) {
                    const float dr = A.dfc_scale * sinc_u(u2);
                    w = make_float4(cutoff_u(u2), dr * dx, dr * dy, dr * dz);
                    live = true;
                }
            }
            const unsigned bm = __ballot_sync(FULL, live);
            if (live) {
                const int k = nlive + __popc(bm & lanemask_lt());
                s_j[warp][k] = j;
                s_w[warp][k] = w;
            }
            nlive += __popc(bm);
        }
        __syncwarp();
        float4 gi[VPL], hi[VPL], acc[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            gi[v] = g4[(size_t)i * F4 + v * LPE + fl];
            hi[v] = h4[(size_t)i * F4 + v * LPE + fl];
            acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float fx = 0.f, fy = 0.f, fz = 0.f;
        for (int e0 = 0; e0 < nlive; e0 += EPI) {
            const int e = e0 + g;
            const bool ok = e < nlive;
            const int j = ok ? s_j[warp][e] : (int)i;
            const float4 w = ok ? s_w[warp][e] : make_float4(0.f, 0.f, 0.f, 0.f);
            float dot = 0.f;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const float4 hj = h4[(size_t)j * F4 + v * LPE + fl];
                const float4 gj = g4[(size_t)j * F4 + v * LPE + fl];
                acc[v].x = fmaf(w.x, gj.x, acc[v].x);
                acc[v].y = fmaf(w.x, gj.y, acc[v].y);
                acc[v].z = fmaf(w.x, gj.z, acc[v].z);
                acc[v].w = fmaf(w.x, gj.w, acc[v].w);
                dot = fmaf(gi[v].x, hj.x, fmaf(gj.x, hi[v].x, dot));
                dot = fmaf(gi[v].y, hj.y, fmaf(gj.y, hi[v].y, dot));
                dot = fmaf(gi[v].z, hj.z, fmaf(gj.z, hi[v].z, dot));
                dot = fmaf(gi[v].w, hj.w, fmaf(gj.w, hi[v].w, dot));
            }
#pragma unroll
            for (int o = 1; o < LPE; o <<= 1) dot += __shfl_xor_sync(FULL, dot, o);
            if (ok) {
                fx = fmaf(dot, w.y, fx);
                fy = fmaf(dot, w.z, fy);
                fz = fmaf(dot, w.w, fz);
            }
        }
        // lane groups hold disjoint edges (sum them); within a group every
        // lane holds the same force but different features
#pragma unroll
        for (int o = LPE; o < 32; o <<= 1) {
            fx += __shfl_xor_sync(FULL, fx, o);
            fy += __shfl_xor_sync(FULL, fy, o);
            fz += __shfl_xor_sync(FULL, fz, o);
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                acc[v].x += __shfl_xor_sync(FULL, acc[v].x, o);
                acc[v].y += __shfl_xor_sync(FULL, acc[v].y, o);
                acc[v].z += __shfl_xor_sync(FULL, acc[v].z, o);
                acc[v].w += __shfl_xor_sync(FULL, acc[v].w, o);
            }
        }
        if (g == 0) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) gf4[(size_t)i * F4 + v * LPE + fl] = acc[v];
        }
        if (lane == 0) {
            A.grad_pos[3 * (size_t)i] = -fx;
            A.grad_pos[3 * (size_t)i + 1] = -fy;
            A.grad_pos[3 * (size_t)i + 2] = -fz;
        }
        __syncwarp();
    }
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
    A.dfc_scale = (float)(-9.8696044010893586188 / (2.0 * (double)rc * (double)rc));
    StageScope sc(ST_BACKWARD, s);
    const int blocks = (int)std::min<long long>(((long long)n + BK_WARPS - 1) / BK_WARPS, (long long)sms * 32);
    switch (F / 4) {
        case 1: edge_backward_kernel<1, 1><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 2: edge_backward_kernel<2, 1><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 4: edge_backward_kernel<2, 2><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 8: edge_backward_kernel<4, 2><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 16: edge_backward_kernel<8, 2><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 32: edge_backward_kernel<16, 2><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        case 64: edge_backward_kernel<32, 2><<<blocks, BK_WARPS * 32, 0, s>>>(A); break;
        default: return TESS_ERR_INVALID_ARG;    // F a multiple of 4 that is not 4 * 2^k
    }
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
    const bool vec4 = (F % 4 == 0) && F <= 256 && aligned(feat, 16) && aligned(out, 16) && cap <= EV_MAXCAP;
    const int vblocks = (int)std::min<long long>(((long long)n + EV_WARPS - 1) / EV_WARPS, (long long)sms * 32);
    bool launched = false;
    if (vec4) {
        launched = true;
        switch (F / 4) {
            case 1: edge_vec4_kernel<1, 1><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 2: edge_vec4_kernel<2, 1><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 4: edge_vec4_kernel<2, 2><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 8: edge_vec4_kernel<4, 2><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 16: edge_vec4_kernel<8, 2><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 32: edge_vec4_kernel<16, 2><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            case 64: edge_vec4_kernel<32, 2><<<vblocks, EV_WARPS * 32, 0, s>>>(A); break;
            default: launched = false; break;
        }
    }
    if (!launched) {
        if ((F % 2 == 0) && aligned(feat, 8) && F >= 64) edge_kernel<2><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
        else edge_kernel<1><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
    }
    count_launch();
    return launch_status();
}

}  // namespace tess
