// Preprocess forward (EWA projection) and backward (2D -> 3D chain rule).
//
// Forward: "4-3DGS训练与优化" section D.4 (Sigma = R S S^T R^T from a unit
// quaternion) and section E.3 (AABB of each projected Gaussian against the
// tile grid); "Gaussian Splatting反向传播的CUDA实现" section 4 (the projection
// whose Jacobian J carries the perspective nonlinearity).
// Backward: the same page, section 4 (2D mean -> 3D mean through the view
// transform and the perspective; dL/dSigma through J; Sigma = R S S^T R^T ->
// scale and rotation), written as one thread per Gaussian.
//
// The forward uses explicit round-to-nearest intrinsics in a fixed order (no
// contraction into FMA): every integer it decides (cull, radius, tile
// rectangle) and the depth bits that order the sort are then reproducible by
// any IEEE fp32 implementation that performs the same operations.

#include <cuda_runtime.h>
#include <math.h>

#include "gs_internal.cuh"
#include "pdl.cuh"

namespace gs {
namespace {

#define ADD __fadd_rn
#define SUB __fsub_rn
#define MUL __fmul_rn
#define DIV __fdiv_rn

constexpr int kPreBlock = 256;

struct Proj {
    float u, v, depth, ca, cb, cc;
    int radius;
    int x0, y0, x1, y1;
    unsigned touched;
};

// Returns false when the Gaussian is culled.
__device__ __forceinline__ bool project(const gs_camera& cam, int TX, int TY, float mx, float my, float mz,
                                        float sx, float sy, float sz, float qw, float qx, float qy, float qz,
                                        Proj& p) {
    const float* W = cam.R;
    const float tx = ADD(ADD(ADD(MUL(W[0], mx), MUL(W[1], my)), MUL(W[2], mz)), cam.t[0]);
    const float ty = ADD(ADD(ADD(MUL(W[3], mx), MUL(W[4], my)), MUL(W[5], mz)), cam.t[1]);
    const float tz = ADD(ADD(ADD(MUL(W[6], mx), MUL(W[7], my)), MUL(W[8], mz)), cam.t[2]);
    if (!(tz > cam.z_near)) return false;

    const float n2 = ADD(ADD(ADD(MUL(qw, qw), MUL(qx, qx)), MUL(qy, qy)), MUL(qz, qz));
    if (!(n2 > 0.0f)) return false;
    const float qn = __fsqrt_rn(n2);
    const float w = DIV(qw, qn), x = DIV(qx, qn), y = DIV(qy, qn), z = DIV(qz, qn);

    const float xx = MUL(x, x), yy = MUL(y, y), zz = MUL(z, z);
    const float xy = MUL(x, y), xz = MUL(x, z), yz = MUL(y, z);
    const float wx = MUL(w, x), wy = MUL(w, y), wz = MUL(w, z);
    float R[3][3];
    R[0][0] = SUB(1.0f, MUL(2.0f, ADD(yy, zz)));
    R[0][1] = MUL(2.0f, SUB(xy, wz));
    R[0][2] = MUL(2.0f, ADD(xz, wy));
    R[1][0] = MUL(2.0f, ADD(xy, wz));
    R[1][1] = SUB(1.0f, MUL(2.0f, ADD(xx, zz)));
    R[1][2] = MUL(2.0f, SUB(yz, wx));
    R[2][0] = MUL(2.0f, SUB(xz, wy));
    R[2][1] = MUL(2.0f, ADD(yz, wx));
    R[2][2] = SUB(1.0f, MUL(2.0f, ADD(xx, yy)));

    const float s[3] = {sx, sy, sz};
    float L[3][3];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int k = 0; k < 3; ++k) L[i][k] = MUL(R[i][k], s[k]);
    float S3[3][3];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = i; j < 3; ++j) {
            S3[i][j] = ADD(ADD(MUL(L[i][0], L[j][0]), MUL(L[i][1], L[j][1])), MUL(L[i][2], L[j][2]));
            S3[j][i] = S3[i][j];
        }

    const float tz2 = MUL(tz, tz);
    const float J[2][3] = {{DIV(cam.fx, tz), 0.0f, DIV(-MUL(cam.fx, tx), tz2)},
                           {0.0f, DIV(cam.fy, tz), DIV(-MUL(cam.fy, ty), tz2)}};
    float M[2][3];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int k = 0; k < 3; ++k)
            M[i][k] = ADD(ADD(MUL(J[i][0], W[k]), MUL(J[i][1], W[3 + k])), MUL(J[i][2], W[6 + k]));
    float T[2][3];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int k = 0; k < 3; ++k)
            T[i][k] = ADD(ADD(MUL(M[i][0], S3[0][k]), MUL(M[i][1], S3[1][k])), MUL(M[i][2], S3[2][k]));
    const float s00 = ADD(ADD(MUL(T[0][0], M[0][0]), MUL(T[0][1], M[0][1])), MUL(T[0][2], M[0][2]));
    const float s01 = ADD(ADD(MUL(T[0][0], M[1][0]), MUL(T[0][1], M[1][1])), MUL(T[0][2], M[1][2]));
    const float s11 = ADD(ADD(MUL(T[1][0], M[1][0]), MUL(T[1][1], M[1][1])), MUL(T[1][2], M[1][2]));
    const float a = ADD(s00, cam.eps2d), b = s01, c = ADD(s11, cam.eps2d);

    const float det = SUB(MUL(a, c), MUL(b, b));
    if (!(det > 0.0f)) return false;
    p.ca = DIV(c, det);
    p.cb = DIV(-b, det);
    p.cc = DIV(a, det);
    const float mid = MUL(0.5f, ADD(a, c));
    const float disc = SUB(MUL(mid, mid), det);
    const float lam = ADD(mid, __fsqrt_rn(disc < 0.0f ? 0.0f : disc));
    p.u = ADD(DIV(MUL(cam.fx, tx), tz), cam.cx);
    p.v = ADD(DIV(MUL(cam.fy, ty), tz), cam.cy);
    if (!isfinite(p.u) || !isfinite(p.v) || isnan(lam)) return false;
    float rr = ceilf(MUL(cam.sigma_mult, __fsqrt_rn(lam)));
    if (!(rr <= 16777216.0f)) rr = 16777216.0f;

    const float ts = (float)kTile;
    auto clampi = [](float v, int hi) -> int {
        if (v < 0.0f) v = 0.0f;
        if (v > (float)hi) v = (float)hi;
        return (int)v;
    };
    p.x0 = clampi(floorf(DIV(SUB(p.u, rr), ts)), TX);
    p.y0 = clampi(floorf(DIV(SUB(p.v, rr), ts)), TY);
    p.x1 = clampi(ceilf(DIV(ADD(p.u, rr), ts)), TX);
    p.y1 = clampi(ceilf(DIV(ADD(p.v, rr), ts)), TY);
    p.touched = (unsigned)((p.x1 - p.x0) * (p.y1 - p.y0));
    if (p.touched == 0) return false;
    p.radius = (int)rr;
    p.depth = tz;
    return true;
}

__global__ void __launch_bounds__(kPreBlock)
k_preprocess_fwd(gs_camera cam, int N, int TX, int TY, const float* __restrict__ means,
                 const float* __restrict__ scales, const float4* __restrict__ quats,
                 const float* __restrict__ opacity, float2* __restrict__ mean2d, float* __restrict__ depth,
                 float4* __restrict__ conic_opacity, int* __restrict__ radius, int4* __restrict__ rect,
                 unsigned* __restrict__ tiles_touched, unsigned* __restrict__ d_num_pairs, WsHeader* hdr,
                 unsigned long long* partials) {
    const int i = blockIdx.x * kPreBlock + threadIdx.x;
    unsigned long long touched = 0;
    if (i < N) {
        const float4 q = quats[i];
        Proj p;
        const bool vis = project(cam, TX, TY, means[3 * i], means[3 * i + 1], means[3 * i + 2], scales[3 * i],
                                 scales[3 * i + 1], scales[3 * i + 2], q.x, q.y, q.z, q.w, p);
        if (vis) {
            mean2d[i] = make_float2(p.u, p.v);
            depth[i] = p.depth;
            conic_opacity[i] = make_float4(p.ca, p.cb, p.cc, opacity[i]);
            radius[i] = p.radius;
            rect[i] = make_int4(p.x0, p.y0, p.x1, p.y1);
            tiles_touched[i] = p.touched;
            touched = p.touched;
        } else {
            mean2d[i] = make_float2(0.0f, 0.0f);
            depth[i] = 0.0f;
            conic_opacity[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            radius[i] = 0;
            rect[i] = make_int4(0, 0, 0, 0);
            tiles_touched[i] = 0;
        }
    }
    // Total pair count: per-block sums, then the last block to finish adds
    // them in block order (deterministic) and resets the ticket.
    __shared__ unsigned long long s_red[kPreBlock / 32];
    __shared__ bool s_last;
    for (int o = 16; o > 0; o >>= 1) touched += __shfl_xor_sync(0xffffffffu, touched, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = touched;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long sum = 0;
        for (int w = 0; w < kPreBlock / 32; ++w) sum += s_red[w];
        partials[blockIdx.x] = sum;
        __threadfence();
        const unsigned t = atomicAdd(&hdr->ticket, 1u);
        s_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    unsigned long long sum = 0;
    for (int b = threadIdx.x; b < (int)gridDim.x; b += kPreBlock)
        sum += ((volatile unsigned long long*)partials)[b];
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long tot = 0;
        for (int w = 0; w < kPreBlock / 32; ++w) tot += s_red[w];
        if (tot > 0xFFFFFFFFull) {
            raise_status(hdr, GS_ERR_OVERFLOW);
            *d_num_pairs = 0xFFFFFFFFu;
        } else {
            *d_num_pairs = (unsigned)tot;
        }
        hdr->ticket = 0;
    }
}

#undef ADD
#undef SUB
#undef MUL
#undef DIV

// ---------------------------------------------------------------------------
// Backward.
// Sigma2 = V V^T + eps I with V = M L, M = J W (2x3), L = R diag(s) (3x3).
// With G2 = dL/dSigma2 (symmetric): dL/dV = 2 G2 V, dL/dM = (dL/dV) L^T,
// dL/dL = M^T (dL/dV).  G2 itself comes from the conic gradient through the
// inverse: G2 = -A Gbar A with A the conic and Gbar the symmetric matrix whose
// off-diagonal is half the gradient w.r.t. the unique entry b.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPreBlock)
k_preprocess_bwd(gs_camera cam, int N, const float* __restrict__ means, const float* __restrict__ scales,
                 const float4* __restrict__ quats, const int* __restrict__ radius,
                 const float4* __restrict__ conic_opacity, const float2* __restrict__ dL_dmean2d,
                 const float4* __restrict__ dL_dconic_opacity, const float* __restrict__ dL_dcolor2d,
                 float* __restrict__ dL_dmeans, float* __restrict__ dL_dscales, float4* __restrict__ dL_dquats,
                 float* __restrict__ dL_dopacity, float* __restrict__ dL_dcolors, float* __restrict__ grad2d_accum,
                 unsigned* __restrict__ vis_count) {
    pdl_enter();
    const int i = blockIdx.x * kPreBlock + threadIdx.x;
    if (i >= N) return;
    // Every load of this Gaussian - inputs and the accumulators read by the
    // += below - is issued here, before the culling test, so that they are
    // in flight together: one memory round trip instead of three (radius,
    // then the inputs, then the accumulators).
    const int rad = radius[i];
    const float mx = means[3 * i], my = means[3 * i + 1], mz = means[3 * i + 2];
    const float4 qv = quats[i];
    const float s[3] = {scales[3 * i], scales[3 * i + 1], scales[3 * i + 2]};
    const float4 co = conic_opacity[i];
    const float4 gco = dL_dconic_opacity[i];
    const float2 gm = dL_dmean2d[i];
    const float gc0 = dL_dcolor2d[3 * i + 0], gc1 = dL_dcolor2d[3 * i + 1], gc2 = dL_dcolor2d[3 * i + 2];
    const float am0 = dL_dmeans[3 * i + 0], am1 = dL_dmeans[3 * i + 1], am2 = dL_dmeans[3 * i + 2];
    const float as0 = dL_dscales[3 * i + 0], as1 = dL_dscales[3 * i + 1], as2 = dL_dscales[3 * i + 2];
    float4 dq = dL_dquats[i];
    const float aop = dL_dopacity[i];
    const float ac0 = dL_dcolors[3 * i + 0], ac1 = dL_dcolors[3 * i + 1], ac2 = dL_dcolors[3 * i + 2];
    const float ga = grad2d_accum ? grad2d_accum[i] : 0.0f;
    const unsigned vc = grad2d_accum ? vis_count[i] : 0u;
    if (rad == 0) return;
    if (grad2d_accum) {
        // densification statistics: |dL/dmean2d| of this view, and one more view
        grad2d_accum[i] = ga + sqrtf(gm.x * gm.x + gm.y * gm.y);
        vis_count[i] = vc + 1u;
    }
    const float* W = cam.R;
    const float tx = W[0] * mx + W[1] * my + W[2] * mz + cam.t[0];
    const float ty = W[3] * mx + W[4] * my + W[5] * mz + cam.t[1];
    const float tz = W[6] * mx + W[7] * my + W[8] * mz + cam.t[2];
    const float qnorm = sqrtf(qv.x * qv.x + qv.y * qv.y + qv.z * qv.z + qv.w * qv.w);
    const float inv_n = 1.0f / qnorm;
    const float w = qv.x * inv_n, x = qv.y * inv_n, y = qv.z * inv_n, z = qv.w * inv_n;
    float R[3][3];
    R[0][0] = 1.f - 2.f * (y * y + z * z);
    R[0][1] = 2.f * (x * y - w * z);
    R[0][2] = 2.f * (x * z + w * y);
    R[1][0] = 2.f * (x * y + w * z);
    R[1][1] = 1.f - 2.f * (x * x + z * z);
    R[1][2] = 2.f * (y * z - w * x);
    R[2][0] = 2.f * (x * z - w * y);
    R[2][1] = 2.f * (y * z + w * x);
    R[2][2] = 1.f - 2.f * (x * x + y * y);

    const float iz = 1.0f / tz;
    const float iz2 = iz * iz;
    const float J00 = cam.fx * iz, J02 = -cam.fx * tx * iz2;
    const float J11 = cam.fy * iz, J12 = -cam.fy * ty * iz2;
    float M[2][3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        M[0][k] = J00 * W[k] + J02 * W[6 + k];
        M[1][k] = J11 * W[3 + k] + J12 * W[6 + k];
    }
    // V = M L with L = R diag(s)
    float V[2][3];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int k = 0; k < 3; ++k) V[r][k] = (M[r][0] * R[0][k] + M[r][1] * R[1][k] + M[r][2] * R[2][k]) * s[k];

    // G2 = -A Gbar A
    const float A00 = co.x, A01 = co.y, A11 = co.z;
    const float g00 = gco.x, g01 = 0.5f * gco.y, g11 = gco.z;
    const float P00 = A00 * g00 + A01 * g01, P01 = A00 * g01 + A01 * g11;
    const float P10 = A01 * g00 + A11 * g01, P11 = A01 * g01 + A11 * g11;
    const float G00 = -(P00 * A00 + P01 * A01);
    const float G01 = -(P00 * A01 + P01 * A11);
    const float G11 = -(P10 * A01 + P11 * A11);

    // dL/dV = 2 G2 V
    float GV[2][3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        GV[0][k] = 2.f * (G00 * V[0][k] + G01 * V[1][k]);
        GV[1][k] = 2.f * (G01 * V[0][k] + G11 * V[1][k]);
    }
    // dL/dL = M^T GV ; dL/dM = GV L^T
    float GL[3][3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int k = 0; k < 3; ++k) GL[r][k] = M[0][r] * GV[0][k] + M[1][r] * GV[1][k];
    float GM[2][3];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int k = 0; k < 3; ++k)
            GM[r][k] = GV[r][0] * R[k][0] * s[0] + GV[r][1] * R[k][1] * s[1] + GV[r][2] * R[k][2] * s[2];
    // dL/dJ = GM W^T (only the four non-zero entries of J depend on t)
    const float GJ00 = GM[0][0] * W[0] + GM[0][1] * W[1] + GM[0][2] * W[2];
    const float GJ02 = GM[0][0] * W[6] + GM[0][1] * W[7] + GM[0][2] * W[8];
    const float GJ11 = GM[1][0] * W[3] + GM[1][1] * W[4] + GM[1][2] * W[5];
    const float GJ12 = GM[1][0] * W[6] + GM[1][1] * W[7] + GM[1][2] * W[8];

    const float iz3 = iz2 * iz;
    float dtx = cam.fx * iz * gm.x - cam.fx * iz2 * GJ02;
    float dty = cam.fy * iz * gm.y - cam.fy * iz2 * GJ12;
    float dtz = -cam.fx * tx * iz2 * gm.x - cam.fy * ty * iz2 * gm.y - cam.fx * iz2 * GJ00 +
                2.f * cam.fx * tx * iz3 * GJ02 - cam.fy * iz2 * GJ11 + 2.f * cam.fy * ty * iz3 * GJ12;
    dL_dmeans[3 * i + 0] = am0 + (W[0] * dtx + W[3] * dty + W[6] * dtz);
    dL_dmeans[3 * i + 1] = am1 + (W[1] * dtx + W[4] * dty + W[7] * dtz);
    dL_dmeans[3 * i + 2] = am2 + (W[2] * dtx + W[5] * dty + W[8] * dtz);

    // scales and rotation from dL/dL
    float GR[3][3];
    const float as[3] = {as0, as1, as2};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        dL_dscales[3 * i + k] = as[k] + (GL[0][k] * R[0][k] + GL[1][k] * R[1][k] + GL[2][k] * R[2][k]);
#pragma unroll
        for (int r = 0; r < 3; ++r) GR[r][k] = GL[r][k] * s[k];
    }
    // d R / d q_hat contracted with GR
    const float dw = 2.f * (-z * GR[0][1] + y * GR[0][2] + z * GR[1][0] - x * GR[1][2] - y * GR[2][0] + x * GR[2][1]);
    const float dx = 2.f * (y * GR[0][1] + z * GR[0][2] + y * GR[1][0] - 2.f * x * GR[1][1] - w * GR[1][2] +
                            z * GR[2][0] + w * GR[2][1] - 2.f * x * GR[2][2]);
    const float dy = 2.f * (-2.f * y * GR[0][0] + x * GR[0][1] + w * GR[0][2] + x * GR[1][0] + z * GR[1][2] -
                            w * GR[2][0] + z * GR[2][1] - 2.f * y * GR[2][2]);
    const float dz = 2.f * (-2.f * z * GR[0][0] - w * GR[0][1] + x * GR[0][2] + w * GR[1][0] - 2.f * z * GR[1][1] +
                            y * GR[1][2] + x * GR[2][0] + y * GR[2][1]);
    // through q_hat = q / |q|
    const float dotp = w * dw + x * dx + y * dy + z * dz;
    dq.x += (dw - w * dotp) * inv_n;
    dq.y += (dx - x * dotp) * inv_n;
    dq.z += (dy - y * dotp) * inv_n;
    dq.w += (dz - z * dotp) * inv_n;
    dL_dquats[i] = dq;
    dL_dopacity[i] = aop + gco.w;
    dL_dcolors[3 * i + 0] = ac0 + gc0;
    dL_dcolors[3 * i + 1] = ac1 + gc1;
    dL_dcolors[3 * i + 2] = ac2 + gc2;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_preprocess_ws_bytes(int N) {
    if (N < 0) return 0;
    const size_t blocks = (size_t)(N + kPreBlock - 1) / kPreBlock + 1;
    return sizeof(WsHeader) + align_up(blocks * sizeof(unsigned long long), 256);
}

extern "C" int gs_preprocess_fwd(const gs_camera* cam, int N, const float* means, const float* scales,
                                 const float* quats, const float* opacity, float* mean2d, float* depth,
                                 float* conic_opacity, int* radius, int* rect, unsigned* tiles_touched,
                                 unsigned* d_num_pairs, void* ws, size_t ws_bytes, void* stream) {
    if (!camera_ok(cam) || N < 0 || !d_num_pairs || !ws) return GS_ERR_INVALID_ARG;
    if (ws_bytes < gs_preprocess_ws_bytes(N) || !aligned(ws, 16)) return GS_ERR_INVALID_ARG;
    if (N > 0) {
        if (!means || !scales || !quats || !opacity || !mean2d || !depth || !conic_opacity || !radius || !rect ||
            !tiles_touched)
            return GS_ERR_INVALID_ARG;
        if (!aligned(quats, 16) || !aligned(conic_opacity, 16) || !aligned(rect, 16) || !aligned(mean2d, 8))
            return GS_ERR_INVALID_ARG;
    }
    const int blocks = (N + kPreBlock - 1) / kPreBlock;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    unsigned long long* partials = reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(ws) + sizeof(WsHeader));
    k_preprocess_fwd<<<blocks > 0 ? blocks : 1, kPreBlock, 0, (cudaStream_t)stream>>>(
        *cam, N, tiles_x(*cam), tiles_y(*cam), means, scales, reinterpret_cast<const float4*>(quats), opacity,
        reinterpret_cast<float2*>(mean2d), depth, reinterpret_cast<float4*>(conic_opacity), radius,
        reinterpret_cast<int4*>(rect), tiles_touched, d_num_pairs, hdr, partials); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

extern "C" int gs_preprocess_bwd(const gs_camera* cam, int N, const float* means, const float* scales,
                                 const float* quats, const int* radius, const float* conic_opacity,
                                 const float* dL_dmean2d, const float* dL_dconic_opacity, const float* dL_dcolor2d,
                                 float* dL_dmeans, float* dL_dscales, float* dL_dquats, float* dL_dopacity,
                                 float* dL_dcolors, float* grad2d_accum, unsigned* vis_count, void* stream) {
    if (!camera_ok(cam) || N < 0) return GS_ERR_INVALID_ARG;
    if ((grad2d_accum == nullptr) != (vis_count == nullptr)) return GS_ERR_INVALID_ARG;
    if (N == 0) return GS_OK;
    if (!means || !scales || !quats || !radius || !conic_opacity || !dL_dmean2d || !dL_dconic_opacity ||
        !dL_dcolor2d || !dL_dmeans || !dL_dscales || !dL_dquats || !dL_dopacity || !dL_dcolors)
        return GS_ERR_INVALID_ARG;
    if (!aligned(quats, 16) || !aligned(conic_opacity, 16) || !aligned(dL_dconic_opacity, 16) ||
        !aligned(dL_dquats, 16) || !aligned(dL_dmean2d, 8))
        return GS_ERR_INVALID_ARG;
    const int blocks = (N + kPreBlock - 1) / kPreBlock;
    launch_pdl(k_preprocess_bwd, blocks, kPreBlock, 0, (cudaStream_t)stream, *cam, N, means, scales,
               reinterpret_cast<const float4*>(quats), radius, reinterpret_cast<const float4*>(conic_opacity),
               reinterpret_cast<const float2*>(dL_dmean2d), reinterpret_cast<const float4*>(dL_dconic_opacity),
               dL_dcolor2d, dL_dmeans, dL_dscales, reinterpret_cast<float4*>(dL_dquats), dL_dopacity, dL_dcolors,
               grad2d_accum, vis_count);
    note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

// ---------------------------------------------------------------------------
// gs_preprocess_fwd_noalloc: the same projection for callers that may not
// allocate device memory at all - a plug-in living inside a host application
// whose allocator owns every device byte, or a per-frame loop where a
// cudaMalloc would synchronise the device and stall the frame.  Such callers
// cannot provide the workspace gs_preprocess_fwd asks for, so this variant
// keeps its scratch (the status/ticket header and one 64-bit partial sum per
// 256 Gaussians) in a fixed array compiled into the library.
// ---------------------------------------------------------------------------
#include <mutex>

namespace gs {
namespace {

constexpr size_t kNoAllocScratchBytes =
    sizeof(WsHeader) + (size_t)(GS_NOALLOC_MAX_GAUSSIANS / kPreBlock) * sizeof(unsigned long long);

// One copy per device that loads the library, resident until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 256;
std::mutex g_noalloc_mutex;
void* g_noalloc_device_addr[kNoAllocMaxDevices];  // device address of the array, per device

// The array's name is only a host-side handle; the device address must be
// looked up with the device current.  Done once per device, on first use.
int noalloc_scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    if (dev < 0 || dev >= kNoAllocMaxDevices) return GS_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_device_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return GS_ERR_CUDA;
        }
        g_noalloc_device_addr[dev] = p;
    }
    *out = g_noalloc_device_addr[dev];
    return GS_OK;
}

}  // namespace
}  // namespace gs

extern "C" int gs_preprocess_fwd_noalloc(const gs_camera* cam, int N, const float* means, const float* scales,
                                         const float* quats, const float* opacity, float* mean2d, float* depth,
                                         float* conic_opacity, int* radius, int* rect, unsigned* tiles_touched,
                                         unsigned* d_num_pairs, void* stream) {
    if (N < 0 || N > GS_NOALLOC_MAX_GAUSSIANS) return GS_ERR_INVALID_ARG;
    if (!camera_ok(cam) || !d_num_pairs) return GS_ERR_INVALID_ARG;
    if (N > 0) {
        if (!means || !scales || !quats || !opacity || !mean2d || !depth || !conic_opacity || !radius || !rect ||
            !tiles_touched)
            return GS_ERR_INVALID_ARG;
        if (!aligned(quats, 16) || !aligned(conic_opacity, 16) || !aligned(rect, 16) || !aligned(mean2d, 8))
            return GS_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    const int rc = noalloc_scratch_address(&scratch);
    if (rc != GS_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    // the header (status word and last-block ticket) must start at zero
    if (cudaMemsetAsync(scratch, 0, sizeof(WsHeader), st) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    const int blocks = (N + kPreBlock - 1) / kPreBlock;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(scratch);
    unsigned long long* partials =
        reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(scratch) + sizeof(WsHeader));
    k_preprocess_fwd<<<blocks > 0 ? blocks : 1, kPreBlock, 0, st>>>(
        *cam, N, tiles_x(*cam), tiles_y(*cam), means, scales, reinterpret_cast<const float4*>(quats), opacity,
        reinterpret_cast<float2*>(mean2d), depth, reinterpret_cast<float4*>(conic_opacity), radius,
        reinterpret_cast<int4*>(rect), tiles_touched, d_num_pairs, hdr, partials); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}
