// Colour from real spherical harmonics, forward and backward.
//
// "Gaussian Splatting反向传播的CUDA实现", section 4: the colour gradient is
// carried to the spherical-harmonics coefficients through the derivative of
// the SH basis, band-limited to a maximum degree.  Here: the orthonormal real
// SH of degree <= 3 in Cartesian form on the unit view direction
// d = normalise(mean - camera centre) (camera centre = -R^T t), coefficients
// ordered k = l^2 + l + m, colour = max(0, sum_k Y_k(d) sh_k + offset) per
// channel; the clamp at 0 passes no gradient where it is active.
// One thread per Gaussian; HBM-bound (16 x 3 coefficients per Gaussian).
//
// Mixed precision ([CB] sections 5 and 7 name half precision as a memory
// optimisation): the *_f16 entry points read the coefficients stored as IEEE
// binary16 (half the bytes of the largest per-Gaussian array) and compute in
// fp32; colours, gradients and the accumulated dL/dsh stay fp32.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kShBlock = 128;
constexpr int kShMaxK = 16;

// Basis values and their partial derivatives w.r.t. (x, y, z) of the unit
// direction (polynomial form; the normalisation is handled by the caller).
struct ShBasis {
    float Y[kShMaxK];
    float dx[kShMaxK], dy[kShMaxK], dz[kShMaxK];
};

__device__ __forceinline__ void sh_basis(float x, float y, float z, int degree, ShBasis& b) {
#pragma unroll
    for (int k = 0; k < kShMaxK; ++k) b.Y[k] = b.dx[k] = b.dy[k] = b.dz[k] = 0.0f;
    b.Y[0] = 0.28209479177387814f;
    if (degree >= 1) {
        const float c1 = 0.4886025119029199f;
        b.Y[1] = c1 * y; b.dy[1] = c1;
        b.Y[2] = c1 * z; b.dz[2] = c1;
        b.Y[3] = c1 * x; b.dx[3] = c1;
    }
    if (degree >= 2) {
        const float a = 1.0925484305920792f, b2 = 0.31539156525252005f, c = 0.5462742152960396f;
        b.Y[4] = a * x * y;             b.dx[4] = a * y;      b.dy[4] = a * x;
        b.Y[5] = a * y * z;             b.dy[5] = a * z;      b.dz[5] = a * y;
        b.Y[6] = b2 * (3.0f * z * z - 1.0f);                 b.dz[6] = 6.0f * b2 * z;
        b.Y[7] = a * x * z;             b.dx[7] = a * z;      b.dz[7] = a * x;
        b.Y[8] = c * (x * x - y * y);   b.dx[8] = 2.0f * c * x; b.dy[8] = -2.0f * c * y;
    }
    if (degree >= 3) {
        const float a = 0.5900435899266435f, bb = 2.890611442640554f, c = 0.4570457994644658f;
        const float d = 0.3731763325901154f, e = 1.445305721320277f;
        const float xx = x * x, yy = y * y, zz = z * z;
        b.Y[9] = a * y * (3.0f * xx - yy);     b.dx[9] = 6.0f * a * x * y;    b.dy[9] = 3.0f * a * (xx - yy);
        b.Y[10] = bb * x * y * z;              b.dx[10] = bb * y * z;          b.dy[10] = bb * x * z;  b.dz[10] = bb * x * y;
        b.Y[11] = c * y * (5.0f * zz - 1.0f);  b.dy[11] = c * (5.0f * zz - 1.0f); b.dz[11] = 10.0f * c * y * z;
        b.Y[12] = d * z * (5.0f * zz - 3.0f);  b.dz[12] = d * (15.0f * zz - 3.0f);
        b.Y[13] = c * x * (5.0f * zz - 1.0f);  b.dx[13] = c * (5.0f * zz - 1.0f); b.dz[13] = 10.0f * c * x * z;
        b.Y[14] = e * z * (xx - yy);           b.dx[14] = 2.0f * e * x * z;    b.dy[14] = -2.0f * e * y * z; b.dz[14] = e * (xx - yy);
        b.Y[15] = a * x * (xx - 3.0f * yy);    b.dx[15] = 3.0f * a * (xx - yy); b.dy[15] = -6.0f * a * x * y;
    }
}

struct ViewDir {
    float x, y, z, inv_norm;
};

__device__ __forceinline__ ViewDir view_dir(const float3 centre, const float* __restrict__ means, int i) {
    const float vx = means[3 * i] - centre.x, vy = means[3 * i + 1] - centre.y, vz = means[3 * i + 2] - centre.z;
    const float inv = rsqrtf(vx * vx + vy * vy + vz * vz);
    return ViewDir{vx * inv, vy * inv, vz * inv, inv};
}

// Each warp owns 32 consecutive Gaussians, whose coefficient rows are one
// contiguous block of 32 * K * 3 floats: the warp moves that block between
// global and shared memory with coalesced accesses, and each lane then reads
// (and, backward, accumulates) its own row in shared memory.
constexpr int kShWarps = kShBlock / 32;
constexpr int kShBwdBlock = 64;  // two row buffers per warp: fewer warps keep it under 48 KiB
constexpr int kShBwdWarps = kShBwdBlock / 32;
constexpr int kShRow = kShMaxK * 3 + 1;  // padded row stride in shared memory, at most

// Rows are stored with an odd stride (K * 3 rounded up to odd), so the 32
// lanes reading "their" row at the same column hit 32 different banks.
__device__ __forceinline__ int row_stride(int K) { return (K * 3) | 1; }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

// The 32 rows of a warp are one contiguous block of rows * K * 3 elements
// (16-byte aligned whenever the array base is, since g0 is a multiple of
// 32).  It moves as 16-byte vectors: every lane issues all its loads before
// its first shared-memory store, so the block costs one memory round trip.
// Blocks that are not whole vectors (K = 1, a ragged last warp, an unaligned
// base) move element by element.
constexpr int kVecBytes = 16;

template <typename T>
__device__ __forceinline__ void warp_load_rows(float* dst, const T* __restrict__ src, int g0, int N, int K) {
    constexpr int E = kVecBytes / sizeof(T);                       // elements per vector
    constexpr int kMaxVec = (32 * kShMaxK * 3 + 32 * E - 1) / (32 * E);  // vectors per lane, at most
    const int lane = threadIdx.x & 31;
    const int rows = min(32, N - g0);
    const int w = K * 3, rs = row_stride(K), total = rows * w;
    const T* s0 = src + (size_t)g0 * w;
    if (total % E == 0 && aligned(s0, kVecBytes)) {
        const int nv = total / E;
        uint4 v[kMaxVec];
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int idx = lane + 32 * j;
            if (idx < nv) v[j] = reinterpret_cast<const uint4*>(s0)[idx];
        }
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int idx = lane + 32 * j;
            if (idx < nv) {
                const T* e = reinterpret_cast<const T*>(&v[j]);
                int r = (idx * E) / w, c = idx * E - r * w;
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    dst[r * rs + c] = to_f32(e[k]);
                    if (++c == w) { c = 0; ++r; }
                }
            }
        }
    } else {
        for (int idx = lane; idx < total; idx += 32) dst[(idx / w) * rs + idx % w] = to_f32(s0[idx]);
    }
}

__device__ __forceinline__ void warp_store_rows(float* __restrict__ dst, const float* src, int g0, int N, int K) {
    constexpr int kMaxVec = (32 * kShMaxK * 3 + 127) / 128;
    const int lane = threadIdx.x & 31;
    const int rows = min(32, N - g0);
    const int w = K * 3, rs = row_stride(K), total = rows * w;
    float* d0 = dst + (size_t)g0 * w;
    if (total % 4 == 0 && aligned(d0, kVecBytes)) {
        const int nv = total / 4;
        float4 v[kMaxVec];
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int idx = lane + 32 * j;
            if (idx < nv) {
                float* e = reinterpret_cast<float*>(&v[j]);
                int r = (idx * 4) / w, c = idx * 4 - r * w;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    e[k] = src[r * rs + c];
                    if (++c == w) { c = 0; ++r; }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxVec; ++j) {
            const int idx = lane + 32 * j;
            if (idx < nv) reinterpret_cast<float4*>(d0)[idx] = v[j];
        }
    } else {
        for (int idx = lane; idx < total; idx += 32) d0[idx] = src[(idx / w) * rs + idx % w];
    }
}

template <typename T>
__global__ void __launch_bounds__(kShBlock)
k_sh_fwd(int N, int degree, int K, float3 centre, float offset, const float* __restrict__ means,
         const T* __restrict__ sh, float* __restrict__ colors) {
    __shared__ float s_sh[kShWarps][32 * kShRow];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g0 = blockIdx.x * kShBlock + warp * 32;
    if (g0 >= N) return;  // whole warp out of range
    warp_load_rows(s_sh[warp], sh, g0, N, K);
    __syncwarp();
    const int i = g0 + lane;
    if (i >= N) return;
    const ViewDir d = view_dir(centre, means, i);
    ShBasis b;
    sh_basis(d.x, d.y, d.z, degree, b);
    const int nk = (degree + 1) * (degree + 1);
    const float* c = s_sh[warp] + lane * row_stride(K);
    float r = 0.0f, g = 0.0f, bl = 0.0f;
#pragma unroll
    for (int k = 0; k < kShMaxK; ++k) {
        if (k < nk) {
            r = fmaf(b.Y[k], c[3 * k], r);
            g = fmaf(b.Y[k], c[3 * k + 1], g);
            bl = fmaf(b.Y[k], c[3 * k + 2], bl);
        }
    }
    colors[3 * i] = fmaxf(r + offset, 0.0f);
    colors[3 * i + 1] = fmaxf(g + offset, 0.0f);
    colors[3 * i + 2] = fmaxf(bl + offset, 0.0f);
}

template <typename T>
__global__ void __launch_bounds__(kShBwdBlock)
k_sh_bwd(int N, int degree, int K, float3 centre, float offset, const float* __restrict__ means,
         const T* __restrict__ sh, const float* __restrict__ dL_dcolors, float* __restrict__ dL_dsh,
         float* __restrict__ dL_dmeans) {
    __shared__ float s_sh[kShBwdWarps][32 * kShRow];
    __shared__ float s_g[kShBwdWarps][32 * kShRow];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g0 = blockIdx.x * kShBwdBlock + warp * 32;
    if (g0 >= N) return;
    warp_load_rows(s_sh[warp], sh, g0, N, K);
    warp_load_rows(s_g[warp], dL_dsh, g0, N, K);
    __syncwarp();
    const int i = g0 + lane;
    if (i < N) {
        const ViewDir d = view_dir(centre, means, i);
        ShBasis b;
        sh_basis(d.x, d.y, d.z, degree, b);
        const int nk = (degree + 1) * (degree + 1);
        const float* c = s_sh[warp] + lane * row_stride(K);
        float* gs = s_g[warp] + lane * row_stride(K);
        // raw colours again, to know where the clamp at 0 is active
        float raw[3] = {offset, offset, offset};
#pragma unroll
        for (int k = 0; k < kShMaxK; ++k)
            if (k < nk)
                for (int ch = 0; ch < 3; ++ch) raw[ch] = fmaf(b.Y[k], c[3 * k + ch], raw[ch]);
        float g[3];
        for (int ch = 0; ch < 3; ++ch) g[ch] = raw[ch] > 0.0f ? dL_dcolors[3 * i + ch] : 0.0f;
        float gx = 0.0f, gy = 0.0f, gz = 0.0f;  // dL/d(direction components)
#pragma unroll
        for (int k = 0; k < kShMaxK; ++k) {
            if (k < nk) {
                gs[3 * k] += b.Y[k] * g[0];
                gs[3 * k + 1] += b.Y[k] * g[1];
                gs[3 * k + 2] += b.Y[k] * g[2];
                const float s2 = c[3 * k] * g[0] + c[3 * k + 1] * g[1] + c[3 * k + 2] * g[2];
                gx = fmaf(b.dx[k], s2, gx);
                gy = fmaf(b.dy[k], s2, gy);
                gz = fmaf(b.dz[k], s2, gz);
            }
        }
        // through d = v / |v| (v = mean - centre): dL/dv = (dL/dd - d (d . dL/dd)) / |v|
        const float dot = d.x * gx + d.y * gy + d.z * gz;
        dL_dmeans[3 * i] += (gx - d.x * dot) * d.inv_norm;
        dL_dmeans[3 * i + 1] += (gy - d.y * dot) * d.inv_norm;
        dL_dmeans[3 * i + 2] += (gz - d.z * dot) * d.inv_norm;
    }
    __syncwarp();
    warp_store_rows(dL_dsh, s_g[warp], g0, N, K);
}

float3 camera_centre(const gs_camera& cam) {
    // x_cam = R x_world + t, so the centre is -R^T t
    float3 c;
    c.x = -(cam.R[0] * cam.t[0] + cam.R[3] * cam.t[1] + cam.R[6] * cam.t[2]);
    c.y = -(cam.R[1] * cam.t[0] + cam.R[4] * cam.t[1] + cam.R[7] * cam.t[2]);
    c.z = -(cam.R[2] * cam.t[0] + cam.R[5] * cam.t[1] + cam.R[8] * cam.t[2]);
    return c;
}

bool sh_args_ok(const gs_camera* cam, int N, int degree, int K) {
    return camera_ok(cam) && N >= 0 && degree >= 0 && degree <= GS_SH_MAX_DEGREE &&
           K >= (degree + 1) * (degree + 1) && K <= kShMaxK;
}

template <typename T>
int sh_fwd(const gs_camera* cam, int N, int degree, int K, const float* means, const T* sh, float offset,
           float* colors, void* stream) {
    if (!sh_args_ok(cam, N, degree, K)) return GS_ERR_INVALID_ARG;
    if (N == 0) return GS_OK;
    if (!means || !sh || !colors) return GS_ERR_INVALID_ARG;
    k_sh_fwd<T><<<(N + kShBlock - 1) / kShBlock, kShBlock, 0, (cudaStream_t)stream>>>(
        N, degree, K, camera_centre(*cam), offset, means, sh, colors); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

template <typename T>
int sh_bwd(const gs_camera* cam, int N, int degree, int K, const float* means, const T* sh, float offset,
           const float* dL_dcolors, float* dL_dsh, float* dL_dmeans, void* stream) {
    if (!sh_args_ok(cam, N, degree, K)) return GS_ERR_INVALID_ARG;
    if (N == 0) return GS_OK;
    if (!means || !sh || !dL_dcolors || !dL_dsh || !dL_dmeans) return GS_ERR_INVALID_ARG;
    k_sh_bwd<T><<<(N + kShBwdBlock - 1) / kShBwdBlock, kShBwdBlock, 0, (cudaStream_t)stream>>>(
        N, degree, K, camera_centre(*cam), offset, means, sh, dL_dcolors, dL_dsh, dL_dmeans); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" int gs_sh_fwd(const gs_camera* cam, int N, int degree, int K, const float* means, const float* sh,
                         float offset, float* colors, void* stream) {
    return sh_fwd<float>(cam, N, degree, K, means, sh, offset, colors, stream);
}

extern "C" int gs_sh_bwd(const gs_camera* cam, int N, int degree, int K, const float* means, const float* sh,
                         float offset, const float* dL_dcolors, float* dL_dsh, float* dL_dmeans, void* stream) {
    return sh_bwd<float>(cam, N, degree, K, means, sh, offset, dL_dcolors, dL_dsh, dL_dmeans, stream);
}

extern "C" int gs_sh_fwd_f16(const gs_camera* cam, int N, int degree, int K, const float* means,
                             const unsigned short* sh, float offset, float* colors, void* stream) {
    if (sh && !aligned(sh, 2)) return GS_ERR_INVALID_ARG;
    return sh_fwd<__half>(cam, N, degree, K, means, reinterpret_cast<const __half*>(sh), offset, colors, stream);
}

extern "C" int gs_sh_bwd_f16(const gs_camera* cam, int N, int degree, int K, const float* means,
                             const unsigned short* sh, float offset, const float* dL_dcolors, float* dL_dsh,
                             float* dL_dmeans, void* stream) {
    if (sh && !aligned(sh, 2)) return GS_ERR_INVALID_ARG;
    return sh_bwd<__half>(cam, N, degree, K, means, reinterpret_cast<const __half*>(sh), offset, dL_dcolors, dL_dsh,
                          dL_dmeans, stream);
}
