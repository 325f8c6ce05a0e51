// Fused optimiser step for the Gaussians' parameters.
//
// "4-3DGS训练与优化" section C.2: Adam with one learning rate per parameter
// group (position, scale, rotation, opacity, colour) and a linear warm-up of
// the position and scale rates.  The step follows Kingma and Ba's Adam:
//   m <- b1 m + (1 - b1) g,  v <- b2 v + (1 - b2) g^2,
//   p <- p - rate (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps).
// The rasterizer consumes activated values (scales = exp(log scales),
// opacity = sigmoid(logit)) and returns gradients w.r.t. them, so the step
// first chains them to the raw parameters, and afterwards writes the new
// activated values for the next frame; the quaternion is renormalised to
// unit length after its update.  One pass over HBM: every element is read
// (parameter, gradient, two moments) and written (parameter, two moments)
// once.

#include <cuda_runtime.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kAdamBlock = 256;

struct AdamRates {
    float rate[5];     // per group, warm-up applied: means, log scales, quats, logit opacity, colours
    float inv_bc1;     // 1 / (1 - b1^t)
    float inv_bc2;     // 1 / (1 - b2^t)
    float b1, b2, eps;
};

__device__ __forceinline__ float adam_update(float p, float g, float& m, float& v, float rate, const AdamRates& r) {
    m = r.b1 * m + (1.0f - r.b1) * g;
    v = r.b2 * v + (1.0f - r.b2) * g * g;
    const float m_hat = m * r.inv_bc1, v_hat = v * r.inv_bc2;
    return p - rate * m_hat / (sqrtf(v_hat) + r.eps);
}

// Work items, in order: 3N position elements, 3N log-scale elements, N
// logit-opacity elements, C*N colour elements (element-wise), then N
// quaternion rows (renormalised together).  Moment layout (m and v alike):
// [means 3N | log scales 3N | quats 4N | opacity N | colours C N].
__global__ void __launch_bounds__(kAdamBlock)
k_adam(int N, int C, AdamRates r, float* __restrict__ means, float* __restrict__ log_scales,
       float4* __restrict__ quats, float* __restrict__ logit_opacity, float* __restrict__ colors,
       const float* __restrict__ g_means, const float* __restrict__ g_scales, const float4* __restrict__ g_quats,
       const float* __restrict__ g_opacity, const float* __restrict__ g_colors, float* __restrict__ m,
       float* __restrict__ v, float* __restrict__ scales_out, float* __restrict__ opacity_out) {
    const size_t n = (size_t)N;
    const size_t e_means = 3 * n, e_scales = 6 * n, e_op = 7 * n, e_col = 7 * n + (size_t)C * n, e_all = e_col + n;
    const size_t o_scales = 3 * n, o_quats = 6 * n, o_op = 10 * n, o_col = 11 * n;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < e_all; i += stride) {
        if (i < e_means) {
            means[i] = adam_update(means[i], g_means[i], m[i], v[i], r.rate[0], r);
        } else if (i < e_scales) {
            const size_t k = i - e_means;
            const float ls = log_scales[k];
            const float g = g_scales[k] * expf(ls);  // d exp(x) / dx
            const float nls = adam_update(ls, g, m[o_scales + k], v[o_scales + k], r.rate[1], r);
            log_scales[k] = nls;
            if (scales_out) scales_out[k] = expf(nls);
        } else if (i < e_op) {
            const size_t k = i - e_scales;
            const float x = logit_opacity[k];
            const float o = 1.0f / (1.0f + expf(-x));
            const float g = g_opacity[k] * o * (1.0f - o);  // d sigmoid(x) / dx
            const float nx = adam_update(x, g, m[o_op + k], v[o_op + k], r.rate[3], r);
            logit_opacity[k] = nx;
            if (opacity_out) opacity_out[k] = 1.0f / (1.0f + expf(-nx));
        } else if (i < e_col) {
            const size_t k = i - e_op;
            colors[k] = adam_update(colors[k], g_colors[k], m[o_col + k], v[o_col + k], r.rate[4], r);
        } else {
            const size_t k = i - e_col;
            float4 q = quats[k];
            const float4 g = g_quats[k];
            float* mq = m + o_quats + 4 * k;
            float* vq = v + o_quats + 4 * k;
            q.x = adam_update(q.x, g.x, mq[0], vq[0], r.rate[2], r);
            q.y = adam_update(q.y, g.y, mq[1], vq[1], r.rate[2], r);
            q.z = adam_update(q.z, g.z, mq[2], vq[2], r.rate[2], r);
            q.w = adam_update(q.w, g.w, mq[3], vq[3], r.rate[2], r);
            const float nn = q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
            if (nn > 0.0f) {
                const float inv = rsqrtf(nn);
                q = make_float4(q.x * inv, q.y * inv, q.z * inv, q.w * inv);
            }
            quats[k] = q;
        }
    }
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" int gs_adam_step(const gs_adam_config* cfg, int step, int N, int C, float* means, float* log_scales,
                            float* quats, float* logit_opacity, float* colors, const float* dL_dmeans,
                            const float* dL_dscales, const float* dL_dquats, const float* dL_dopacity,
                            const float* dL_dcolors, float* m, float* v, float* scales, float* opacity,
                            void* stream) {
    if (!cfg || step < 1 || N < 0 || C < 0) return GS_ERR_INVALID_ARG;
    if (!(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f && cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f && cfg->eps >= 0.0f))
        return GS_ERR_INVALID_ARG;
    if (N == 0) return GS_OK;
    if (!means || !log_scales || !quats || !logit_opacity || (C > 0 && !colors) || !dL_dmeans || !dL_dscales ||
        !dL_dquats || !dL_dopacity || (C > 0 && !dL_dcolors) || !m || !v)
        return GS_ERR_INVALID_ARG;
    if (!aligned(quats, 16) || !aligned(dL_dquats, 16)) return GS_ERR_INVALID_ARG;
    AdamRates r;
    const double warm = cfg->warmup_steps > 0 ? (step < cfg->warmup_steps ? (double)step / cfg->warmup_steps : 1.0)
                                              : 1.0;
    const float lr[5] = {cfg->lr_means, cfg->lr_scales, cfg->lr_quats, cfg->lr_opacity, cfg->lr_colors};
    for (int k = 0; k < 5; ++k) r.rate[k] = (float)(lr[k] * (k < 2 ? warm : 1.0));
    r.inv_bc1 = (float)(1.0 / (1.0 - pow((double)cfg->beta1, step)));
    r.inv_bc2 = (float)(1.0 / (1.0 - pow((double)cfg->beta2, step)));
    r.b1 = cfg->beta1;
    r.b2 = cfg->beta2;
    r.eps = cfg->eps;
    const size_t items = (size_t)N * (8 + (size_t)C);
    size_t blocks = (items + kAdamBlock - 1) / kAdamBlock;
    if (blocks > 148u * 16u) blocks = 148u * 16u;
    k_adam<<<(unsigned)blocks, kAdamBlock, 0, (cudaStream_t)stream>>>(
        N, C, r, means, log_scales, reinterpret_cast<float4*>(quats), logit_opacity, colors, dL_dmeans, dL_dscales,
        reinterpret_cast<const float4*>(dL_dquats), dL_dopacity, dL_dcolors, m, v, scales, opacity); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}
