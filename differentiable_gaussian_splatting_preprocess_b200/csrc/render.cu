// Tile compositing, forward and backward.
//
// Forward: the rendering equation C = sum_i c_i a_i prod_{j<i} (1 - a_j) of
// "3D高斯散射中的反向传播链式求梯度", with a_i = min(0.99, sigma_i G_i) and
// G_i = exp(-1/2 d^T A d) ("Gaussian Splatting反向传播的CUDA实现", section 2),
// evaluated per 16x16 tile with the tile's Gaussians staged through shared
// memory in batches ("4-3DGS训练与优化", section E.3: tiles are independent).
//
// Backward: the reverse traversal of "Gaussian Splatting反向传播的CUDA实现",
// section 3: start from the forward's final transmittance, walk the tile's
// list from the last contributor towards the front, recover T <- T / (1 - a),
// and accumulate dL/dcolor = T a dL/dC and dL/da = T (c - C_behind) . dL/dC
// (section 2's table), then through G to the conic and the 2D mean.
// Per-Gaussian partial gradients are reduced across the warp and across the
// CTA before any global atomic, so a (tile, Gaussian) pair costs at most one
// float2, one float4 and three float atomics.

#include <cuda_runtime.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kBlock = kTilePixels;  // one thread per pixel of a 16x16 tile

__global__ void __launch_bounds__(kBlock)
k_render_fwd(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
             const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
             const float* __restrict__ colors, float* __restrict__ image, float* __restrict__ final_T,
             unsigned* __restrict__ n_contrib) {
    __shared__ float2 s_xy[kBlock];
    __shared__ float4 s_co[kBlock];
    __shared__ float4 s_col[kBlock];
    const int tile = blockIdx.x;
    const int x = (tile % TX) * kTile + (threadIdx.x & (kTile - 1));
    const int y = (tile / TX) * kTile + (threadIdx.x / kTile);
    const bool inside = x < cam.width && y < cam.height;
    const float px = (float)x + 0.5f, py = (float)y + 0.5f;
    const uint2 rg = ranges[tile];
    const float amax = cam.alpha_max, amin = cam.alpha_min, tmin = cam.T_min;

    float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
    unsigned last = 0;
    bool done = !inside;
    for (unsigned b = rg.x; b < rg.y; b += kBlock) {
        if (__syncthreads_count(done) == kBlock) break;
        const unsigned k = b + threadIdx.x;
        if (k < rg.y) {
            const unsigned j = ids[k];
            s_xy[threadIdx.x] = mean2d[j];
            s_co[threadIdx.x] = conic_opacity[j];
            s_col[threadIdx.x] = make_float4(colors[3 * j], colors[3 * j + 1], colors[3 * j + 2], 0.0f);
        }
        __syncthreads();
        const int n = min((unsigned)kBlock, rg.y - b);
        if (!done) {
            for (int jj = 0; jj < n; ++jj) {
                Term e;
                if (!eval_term(px, py, s_xy[jj], s_co[jj], amax, amin, e)) continue;
                const float Tn = __fmul_rn(T, __fsub_rn(1.0f, e.alpha));
                if (Tn < tmin) {
                    done = true;
                    break;
                }
                const float w = e.alpha * T;
                const float4 c = s_col[jj];
                C0 = fmaf(c.x, w, C0);
                C1 = fmaf(c.y, w, C1);
                C2 = fmaf(c.z, w, C2);
                T = Tn;
                last = b - rg.x + jj + 1;
            }
        }
    }
    if (inside) {
        const size_t pix = (size_t)y * cam.width + x;
        const size_t plane = (size_t)cam.width * cam.height;
        image[pix] = fmaf(T, cam.bg[0], C0);
        image[plane + pix] = fmaf(T, cam.bg[1], C1);
        image[2 * plane + pix] = fmaf(T, cam.bg[2], C2);
        final_T[pix] = T;
        n_contrib[pix] = last;
    }
}

// Butterfly reduction of 8 values across a warp in 9 shuffles: afterwards
// lanes 4i..4i+3 hold the warp sum of value i.
__device__ __forceinline__ float reduce8(float v[8], int lane) {
    const bool b4 = lane & 16;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? v[i] : v[i + 4];
        const float keep = b4 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    const bool b3 = lane & 8;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? v[i] : v[i + 2];
        const float keep = b3 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const bool b2 = lane & 4;
    {
        const float send = b2 ? v[0] : v[1];
        const float keep = b2 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

constexpr int kGradStride = 9;  // floats per staged Gaussian in shared memory

__global__ void __launch_bounds__(kBlock)
k_render_bwd(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
             const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
             const float* __restrict__ colors, const float* __restrict__ final_T,
             const unsigned* __restrict__ n_contrib, const float* __restrict__ dL_dimage,
             float2* __restrict__ dL_dmean2d, float4* __restrict__ dL_dconic_opacity,
             float* __restrict__ dL_dcolor) {
    __shared__ unsigned s_id[kBlock];
    __shared__ float2 s_xy[kBlock];
    __shared__ float4 s_co[kBlock];
    __shared__ float4 s_col[kBlock];
    __shared__ float s_grad[kBlock * kGradStride];
    __shared__ unsigned s_max[kBlock / 32];

    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int x = (tile % TX) * kTile + (threadIdx.x & (kTile - 1));
    const int y = (tile / TX) * kTile + (threadIdx.x / kTile);
    const bool inside = x < cam.width && y < cam.height;
    const float px = (float)x + 0.5f, py = (float)y + 0.5f;
    const uint2 rg = ranges[tile];
    const float amax = cam.alpha_max, amin = cam.alpha_min;

    const size_t pix = (size_t)y * cam.width + x;
    const size_t plane = (size_t)cam.width * cam.height;
    float T = 0.0f, g0 = 0.0f, g1 = 0.0f, g2 = 0.0f;
    unsigned last = 0;
    if (inside) {
        T = final_T[pix];
        last = n_contrib[pix];
        g0 = dL_dimage[pix];
        g1 = dL_dimage[plane + pix];
        g2 = dL_dimage[2 * plane + pix];
    }
    float S0 = cam.bg[0], S1 = cam.bg[1], S2 = cam.bg[2];

    // furthest list position any pixel of the tile blended
    const unsigned wmax = __reduce_max_sync(0xffffffffu, last);
    if (lane == 0) s_max[threadIdx.x >> 5] = wmax;
    for (int i = threadIdx.x; i < kBlock * kGradStride; i += kBlock) s_grad[i] = 0.0f;
    __syncthreads();
    unsigned max_last = 0;
#pragma unroll
    for (int w = 0; w < kBlock / 32; ++w) max_last = max(max_last, s_max[w]);
    max_last = min(max_last, rg.y - rg.x);  // stay inside the tile's list

    for (int top = (int)max_last; top > 0; top -= kBlock) {
        const int pos = top - 1 - (int)threadIdx.x;
        if (pos >= 0) {
            const unsigned j = ids[rg.x + pos];
            s_id[threadIdx.x] = j;
            s_xy[threadIdx.x] = mean2d[j];
            s_co[threadIdx.x] = conic_opacity[j];
            s_col[threadIdx.x] = make_float4(colors[3 * j], colors[3 * j + 1], colors[3 * j + 2], 0.0f);
        }
        __syncthreads();
        const int n = min(kBlock, top);
        for (int jj = 0; jj < n; ++jj) {
            const int p = top - 1 - jj;
            Term e;
            const float4 co = s_co[jj];
            bool contrib = p < (int)last;
            if (contrib) contrib = eval_term(px, py, s_xy[jj], co, amax, amin, e);
            if (!__any_sync(0xffffffffu, contrib)) continue;
            float v[8];
            float vcol2 = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
            if (contrib) {
                T = __fdividef(T, 1.0f - e.alpha);
                const float4 c = s_col[jj];
                const float wgt = e.alpha * T;
                v[5] = wgt * g0;  // dL/dcolor
                v[6] = wgt * g1;
                vcol2 = wgt * g2;
                const float dLda = ((c.x - S0) * g0 + (c.y - S1) * g1 + (c.z - S2) * g2) * T;
                const float om = 1.0f - e.alpha;
                S0 = e.alpha * c.x + om * S0;
                S1 = e.alpha * c.y + om * S1;
                S2 = e.alpha * c.z + om * S2;
                // exact derivative of min(alpha_max, sigma G): zero while capped
                const bool free = e.at <= amax;
                const float dLdsig = free ? e.G * dLda : 0.0f;
                const float h = free ? e.G * co.w * dLda : 0.0f;  // dL/dpower
                const float dx = e.dx, dy = e.dy;
                v[0] = (co.x * dx + co.y * dy) * h;  // dL/du
                v[1] = (co.y * dx + co.z * dy) * h;  // dL/dv
                v[2] = -0.5f * dx * dx * h;          // dL/da
                v[3] = -dx * dy * h;                 // dL/db
                v[4] = -0.5f * dy * dy * h;          // dL/dc
                v[7] = dLdsig;                       // dL/dopacity
            }
            const float r8 = reduce8(v, lane);
            float r9 = vcol2;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r9 += __shfl_xor_sync(0xffffffffu, r9, o);
            // lanes 4i hold value i (i < 8); lane 1 holds the ninth
            float* sg = s_grad + jj * kGradStride;
            if ((lane & 3) == 0) atomicAdd(sg + (lane >> 2), r8);
            if (lane == 1) atomicAdd(sg + 8, r9);
        }
        __syncthreads();
        // flush this batch: one set of global atomics per (tile, Gaussian)
        if (threadIdx.x < n) {
            float* sg = s_grad + threadIdx.x * kGradStride;
            const float a0 = sg[0], a1 = sg[1], a2 = sg[2], a3 = sg[3], a4 = sg[4];
            const float a5 = sg[5], a6 = sg[6], a7 = sg[7], a8 = sg[8];
            const bool any = (a0 != 0.f) | (a1 != 0.f) | (a2 != 0.f) | (a3 != 0.f) | (a4 != 0.f) | (a5 != 0.f) |
                             (a6 != 0.f) | (a7 != 0.f) | (a8 != 0.f);
            if (any) {
                const unsigned j = s_id[threadIdx.x];
                atomicAdd(&dL_dmean2d[j], make_float2(a0, a1));
                atomicAdd(&dL_dconic_opacity[j], make_float4(a2, a3, a4, a7));
                atomicAdd(&dL_dcolor[3 * j + 0], a5);
                atomicAdd(&dL_dcolor[3 * j + 1], a6);
                atomicAdd(&dL_dcolor[3 * j + 2], a8);
            }
#pragma unroll
            for (int i = 0; i < kGradStride; ++i) sg[i] = 0.0f;
        }
        __syncthreads();
    }
}

__global__ void k_zero(float* __restrict__ a, size_t na, float* __restrict__ b, size_t nb, float* __restrict__ c,
                       size_t nc) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < na; i += stride) a[i] = 0.0f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += stride) b[i] = 0.0f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nc; i += stride) c[i] = 0.0f;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" int gs_render_fwd(const gs_camera* cam, const unsigned* ranges, const unsigned* ids, const float* mean2d,
                             const float* conic_opacity, const float* colors, float* image, float* final_T,
                             unsigned* n_contrib, void* stream) {
    if (!camera_ok(cam) || !ranges || !image || !final_T || !n_contrib) return GS_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || (conic_opacity && !aligned(conic_opacity, 16)) || (mean2d && !aligned(mean2d, 8)))
        return GS_ERR_INVALID_ARG;
    const int TX = tiles_x(*cam), T = TX * tiles_y(*cam);
    k_render_fwd<<<T, kBlock, 0, (cudaStream_t)stream>>>(
        *cam, TX, reinterpret_cast<const uint2*>(ranges), ids, reinterpret_cast<const float2*>(mean2d),
        reinterpret_cast<const float4*>(conic_opacity), colors, image, final_T, n_contrib);
    GS_LAUNCH_CHECK();
    return GS_OK;
}

extern "C" int gs_render_bwd(const gs_camera* cam, int N, const unsigned* ranges, const unsigned* ids,
                             const float* mean2d, const float* conic_opacity, const float* colors,
                             const float* final_T, const unsigned* n_contrib, const float* dL_dimage,
                             float* dL_dmean2d, float* dL_dconic_opacity, float* dL_dcolor, void* stream) {
    if (!camera_ok(cam) || N < 0 || !ranges || !final_T || !n_contrib || !dL_dimage) return GS_ERR_INVALID_ARG;
    if (N > 0 && (!dL_dmean2d || !dL_dconic_opacity || !dL_dcolor)) return GS_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || (conic_opacity && !aligned(conic_opacity, 16)) || (mean2d && !aligned(mean2d, 8)) ||
        (dL_dmean2d && !aligned(dL_dmean2d, 8)) || (dL_dconic_opacity && !aligned(dL_dconic_opacity, 16)))
        return GS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (N > 0) {
        size_t work = (size_t)N * 4;
        int blocks = (int)((work + 255) / 256);
        if (blocks > 148 * 8) blocks = 148 * 8;
        k_zero<<<blocks, 256, 0, st>>>(dL_dmean2d, (size_t)N * 2, dL_dconic_opacity, (size_t)N * 4, dL_dcolor,
                                       (size_t)N * 3);
        GS_LAUNCH_CHECK();
    }
    const int TX = tiles_x(*cam), T = TX * tiles_y(*cam);
    k_render_bwd<<<T, kBlock, 0, st>>>(*cam, TX, reinterpret_cast<const uint2*>(ranges), ids,
                                       reinterpret_cast<const float2*>(mean2d),
                                       reinterpret_cast<const float4*>(conic_opacity), colors, final_T, n_contrib,
                                       dL_dimage, reinterpret_cast<float2*>(dL_dmean2d),
                                       reinterpret_cast<float4*>(dL_dconic_opacity), dL_dcolor);
    GS_LAUNCH_CHECK();
    return GS_OK;
}
