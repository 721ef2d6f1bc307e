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
    float rc, inv_rc;
};

__device__ __forceinline__ float min_image_f(float d, float L) {
    if (d > 0.5f * L) return d - L;
    if (d < -0.5f * L) return d + L;
    return d;
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
                    const float r = sqrtf(fmaf(dz, dz, fmaf(dy, dy, dx * dx)));
                    fc = r < A.rc ? 0.5f * (cospif(r * A.inv_rc) + 1.0f) : 0.0f;
                    if (fc0 == 0 && edges) {
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
    A.inv_rc = 1.0f / rc;
    StageScope sc(ST_EDGE, s);
    const long long rows_blocks = ((long long)n + EDGE_WARPS - 1) / EDGE_WARPS;
    const int blocks = (int)std::min<long long>(rows_blocks, (long long)sms * 64);
    const bool vec2 = (F % 2 == 0) && aligned(feat, 8) && F >= 64;
    if (vec2) edge_kernel<2><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
    else edge_kernel<1><<<blocks, EDGE_WARPS * 32, 0, s>>>(A);
    count_launch();
    return launch_status();
}

}  // namespace tess
