/*
 * gs.h - C ABI of the B200 tile rasterizer for differentiable 3D Gaussian
 * Splatting: preprocess, binning, compositing, and both backward stages.
 *
 * Sources of the operations (page title, section):
 *   [CR]  "3D高斯散射中的反向传播链式求梯度" - the rendering equation
 *         C = sum_i c_i a_i prod_{j<i} (1 - a_j) and the mean gradient
 *         dG/dmu = G Sigma^-1 (x - mu).
 *   [CB]  "Gaussian Splatting反向传播的CUDA实现" - section 1 (the backward
 *         reuses the forward's sorted list, tile ranges and final
 *         transmittance, with no dynamic allocation), section 2 (a_i =
 *         min(0.99, sigma_i G_i), G_i = exp(-1/2 d^T A d) and the gradient
 *         table), section 3 (reverse per-pixel traversal from the final
 *         transmittance, T <- T / (1 - a), last contributor), section 4
 *         (2D -> 3D gradients: dL/dSigma through J, Sigma = R S S^T R^T).
 *   [TR]  "4-3DGS训练与优化" - section D.4 (covariance from a unit quaternion
 *         and scales) and section E.3 (tile rasterisation: AABB cull per
 *         tile, depth sort, splat in order, tiles independent).
 *
 * Conventions common to every entry point
 *   - Every pointer argument is DEVICE memory unless stated otherwise; the
 *     caller allocates and owns all of it.  The library never allocates and
 *     never frees.
 *   - Every call only enqueues work on `stream` (0 = legacy default stream)
 *     and returns; no call synchronises except gs_read_status().
 *   - Argument errors are detected on the host and returned immediately as
 *     GS_ERR_INVALID_ARG with nothing enqueued.  Launch failures return
 *     GS_ERR_CUDA.  Conditions found on the device (a pair count above the
 *     caller's capacity, a bounded wait that ran out) are OR-ed into a sticky
 *     status word at the start of the workspace `ws`; read it with
 *     gs_read_status() and clear it with gs_clear_status().
 *   - Layouts are dense, row-major, fp32 unless stated: means [N,3],
 *     scales [N,3] (linear, already activated), quats [N,4] as (w, x, y, z)
 *     (any non-zero norm; normalised inside), opacity [N] (already
 *     activated, in (0, 1]), colors [N,3] RGB.  Images are channel-major
 *     [3, H, W].
 *   - Pixel (x, y) has its centre at (x + 0.5, y + 0.5).  Tiles are 16 x 16
 *     pixels, numbered row-major: tile = ty * ceil(W/16) + tx.
 *   - A Gaussian is "culled" when it is behind the near plane, has a zero
 *     quaternion, a non-positive 2D determinant, a non-finite projection, or
 *     a tile rectangle outside the image.  Culled Gaussians get radius 0,
 *     tiles_touched 0, all-zero 2D outputs and exactly zero gradients.
 */
#ifndef GS_H
#define GS_H

#include <stddef.h>

#if defined(__GNUC__)
#define GS_API __attribute__((visibility("default")))
#else
#define GS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define GS_OK 0
#define GS_ERR_INVALID_ARG 1   /* bad pointer, size or parameter (host check) */
#define GS_ERR_CAPACITY 2      /* device: pair count above the caller's capacity */
#define GS_ERR_TIMEOUT 4       /* device: a bounded wait gave up */
#define GS_ERR_CUDA 8          /* a CUDA launch or copy failed */
#define GS_ERR_UNIMPLEMENTED 16
#define GS_ERR_OVERFLOW 32     /* device: pair count does not fit in 32 bits */
#define GS_ERR_INDEX 64        /* device, debug build only: an index check failed (the access was skipped) */

/* Stages for gs_workspace_bytes(). */
#define GS_STAGE_PREPROCESS_FWD 0
#define GS_STAGE_BIN_SORT 1

#define GS_TILE 16

/* Pinhole camera and rasterizer parameters, passed by host pointer and read
 * during the call (the record may be reused after the call returns). */
typedef struct gs_camera {
    int width, height;  /* image size in pixels, each in [1, 65536] */
    int tile;           /* must be GS_TILE (16) */
    float fx, fy;       /* focal lengths in pixels */
    float cx, cy;       /* principal point in pixels (cx = W/2 is the centre) */
    float R[9];         /* world -> camera rotation, row-major: x_c = R x_w + t */
    float t[3];
    float z_near;       /* cull when the camera-space depth is not > z_near */
    float eps2d;        /* low-pass dilation added to the 2D covariance diagonal (px^2) */
    float alpha_max;    /* opacity cap; 0.99 in [CB] section 2 */
    float alpha_min;    /* terms with alpha below this are skipped (1/255 default) */
    float T_min;        /* a pixel stops before the term that would take T below this */
    float sigma_mult;   /* support radius = ceil(sigma_mult * sqrt(lambda_max)) */
    float bg[3];        /* background colour, composited with the final T */
} gs_camera;

/* Library version as (major << 16) | minor. */
GS_API int gs_version(void);

/* Number of kernels this library has launched in this process so far (all
 * entry points, all streams, all threads).  Host-side count, taken when each
 * launch is issued; a diagnostic for counting launches per frame.  Never
 * fails. */
GS_API unsigned long long gs_launch_count(void);

/* Human-readable text for a status code or a combination of flags. */
GS_API const char* gs_status_string(int status);

/* Bytes of workspace `ws` a stage needs.  `capacity` is the number of
 * (tile, Gaussian) pairs the caller's buffers can hold (GS_STAGE_BIN_SORT);
 * it is ignored for GS_STAGE_PREPROCESS_FWD.  One buffer of the larger size
 * may serve both stages.  A new workspace must be zero-filled once before
 * its first use (e.g. cudaMemsetAsync); every call leaves it ready for the
 * next.  Returns 0 for invalid arguments. */
GS_API size_t gs_workspace_bytes(int stage, int N, unsigned capacity, int width, int height);

/* Copy the sticky device status word of `ws` to *status (host), waiting for
 * `stream` to finish.  The only synchronising call. */
GS_API int gs_read_status(const void* ws, int* status, void* stream);

/* Enqueue a reset of the status word of `ws` to GS_OK. */
GS_API int gs_clear_status(void* ws, void* stream);

/*
 * Debug build (libgs_debug.so: the same sources compiled with GS_DEBUG; no
 * counterpart on the pages, a tool for checking this library).  Before every
 * gather by a Gaussian id or a sorted-list position, and before every write of
 * a sorted-list entry, its kernels check the index against the limits set
 * here (id < n_gauss, list position < capacity); a failed check skips the
 * access and ORs GS_ERR_INDEX into a device-wide debug word instead of
 * touching memory.  Tile indices come from the launch grid and the ranges;
 * the ranges are checked against the capacity.
 *
 * gs_debug_configure - set the limits (and clear the debug word); blocks
 *   until done.  Until it is first called every limit is unbounded.
 * gs_debug_read - copy the debug word to *flags (host), after waiting for
 *   all work on the device; with `clear` != 0 also reset it.
 * In the release library (libgs.so) both return GS_ERR_UNIMPLEMENTED and
 *   *flags is set to 0.
 */
GS_API int gs_debug_configure(unsigned n_gauss, unsigned capacity);
GS_API int gs_debug_read(int* flags, int clear);

/*
 * gs_preprocess_fwd - EWA projection of N 3D Gaussians ([TR] D.4, E.3; [CB] 4).
 *   Per Gaussian: t = R mu + t_cam; q_hat = q / |q|; Sigma3 = (R_q S)(R_q S)^T;
 *   J = pinhole Jacobian at t; Sigma2 = (J R) Sigma3 (J R)^T + eps2d I;
 *   conic = Sigma2^-1; radius = ceil(sigma_mult sqrt(lambda_max(Sigma2)));
 *   (u, v) = (fx tx / tz + cx, fy ty / tz + cy); tile rectangle
 *   [floor((u - r)/16), ceil((u + r)/16)) x [floor((v - r)/16), ceil((v + r)/16))
 *   clamped to the tile grid; tiles_touched = its area; depth = tz.
 *   These values are computed with one IEEE rounding per operation in a fixed
 *   order, so that integer outcomes are reproducible on any IEEE machine.
 * Outputs (device): mean2d [N,2] = (u, v); depth [N]; conic_opacity [N,4] =
 *   (a, b, c, opacity) of the quadratic form a dx^2 + 2 b dx dy + c dy^2;
 *   radius [N] int32; rect [N,4] int32 = (x0, y0, x1, y1) in tiles;
 *   tiles_touched [N] uint32; *d_num_pairs (one uint32) = total pairs P.
 *   If P does not fit in 32 bits, *d_num_pairs = 0xFFFFFFFF and
 *   GS_ERR_OVERFLOW is raised in the status word.
 * ws: >= gs_workspace_bytes(GS_STAGE_PREPROCESS_FWD, N, 0, W, H) bytes,
 *   16-byte aligned.  N = 0 is valid (P = 0).
 */
GS_API int gs_preprocess_fwd(const gs_camera* cam, int N, const float* means, const float* scales,
                      const float* quats, const float* opacity, float* mean2d, float* depth,
                      float* conic_opacity, int* radius, int* rect, unsigned* tiles_touched,
                      unsigned* d_num_pairs, void* ws, size_t ws_bytes, void* stream);

/*
 * gs_preprocess_fwd_noalloc - gs_preprocess_fwd for callers that cannot
 *   allocate device memory (no counterpart on the pages: it is a packaging
 *   variant, not a step of the method).  Examples: a plug-in inside a host
 *   application whose allocator owns all device memory, or a per-frame loop
 *   where a cudaMalloc would synchronise the device.  Same arguments, outputs
 *   and arithmetic as gs_preprocess_fwd, without `ws`: the scratch lives in a
 *   fixed array inside the library (256 bytes + 8 bytes per 256 Gaussians,
 *   about 512 KiB), held on every device that loads the library until the
 *   process exits.
 * Limits and behaviour:
 *   - N > GS_NOALLOC_MAX_GAUSSIANS (or N < 0) returns GS_ERR_INVALID_ARG and
 *     enqueues nothing.
 *   - The first call on a device looks up the array's device address with
 *     that device current (once per device); make that first call before any
 *     stream capture.
 *   - Calls allocate nothing (no cudaMalloc, cudaFree or allocating library
 *     routine).  Each call clears the scratch header on `stream` first.
 *   - Every call on a device shares the one array: calls that overlap on the
 *     GPU (e.g. on two streams at once) race and give wrong pair counts.
 *     Serialise them, or use gs_preprocess_fwd with one workspace each.
 *   - A pair count that does not fit in 32 bits is reported only through
 *     *d_num_pairs = 0xFFFFFFFF (there is no caller-visible status word).
 */
#define GS_NOALLOC_MAX_GAUSSIANS (1 << 24)
GS_API int gs_preprocess_fwd_noalloc(const gs_camera* cam, int N, const float* means, const float* scales,
                      const float* quats, const float* opacity, float* mean2d, float* depth,
                      float* conic_opacity, int* radius, int* rect, unsigned* tiles_touched,
                      unsigned* d_num_pairs, void* stream);

/*
 * gs_bin_sort - tile binning and (tile, depth) sort ([TR] E.3; [CB] 1, 3).
 *   Produces, for every tile, the ids of the Gaussians whose rectangle
 *   contains it, in increasing (depth, id) order, concatenated in tile
 *   order.  The order is exactly that of a sort of the 64-bit keys
 *   (tile << 32 | float_bits(depth)) with ties broken by id.
 * Inputs: depth, rect, tiles_touched from gs_preprocess_fwd; d_num_pairs =
 *   device pointer to P (read on the device, so no host round trip is
 *   needed); capacity = host-side size of `ids` (and of `keys`) in elements.
 * Outputs: ids [capacity] (first P valid); ranges [T,2] uint32 with
 *   ranges[t] = [start, end) into ids, (0, 0) for an empty tile, where
 *   T = ceil(W/16) * ceil(H/16); keys [capacity] uint64 (optional: pass NULL
 *   to skip writing them) with keys[k] = tile << 32 | float_bits(depth[ids[k]]).
 * If P > capacity, GS_ERR_CAPACITY is raised in the status word, every range
 *   is (0, 0) and ids/keys are not written (the caller retries with a larger
 *   capacity).
 * ws: >= gs_workspace_bytes(GS_STAGE_BIN_SORT, N, capacity, W, H) bytes.
 */
GS_API int gs_bin_sort(const gs_camera* cam, int N, const float* depth, const int* rect,
                const unsigned* tiles_touched, const unsigned* d_num_pairs, unsigned capacity,
                unsigned* ids, unsigned* ranges, unsigned long long* keys, void* ws, size_t ws_bytes,
                void* stream);

/*
 * gs_render_fwd - front-to-back compositing per 16x16 tile ([CR] rendering
 *   equation; [CB] 2, 3).  Per pixel p, over its tile's list in order:
 *   d = p - (u, v); power = -1/2 (a dx^2 + c dy^2) - b dx dy (skip if > 0);
 *   alpha = min(alpha_max, opacity exp(power)) (skip if < alpha_min);
 *   stop before a term with T (1 - alpha) < T_min; otherwise
 *   C += color alpha T, T *= (1 - alpha).  Finally C += T bg.
 * Outputs: image [3,H,W]; final_T [H,W]; n_contrib [H,W] uint32 = list
 *   position (within the tile) of the last blended term plus one.
 * colors [N,3] are indexed by the ids in `ids`.
 * contrib_mask (optional, may be NULL; mask_words words, a multiple of 4 and
 *   at least GS_ORDER_WORDS(T) + 4) is the forward's record for gs_render_bwd,
 *   in two parts:
 *   - words [0, GS_ORDER_WORDS(T)): the dispatch-order block.  Words [0, 4T)
 *     receive, per 8x8 quadrant q of tile t, the number of list positions
 *     blended into at least one of its pixels (word 4t + q); words [4T, 8T)
 *     receive the order in which gs_render_bwd dispatches those 4T quadrants
 *     (most blended first); words [8T, 9T) the order in which this call
 *     dispatched its tiles (longest list first); words from 9T on hold the
 *     per-partition counts of quadrants by work class (256 words for each
 *     2048 quadrants) that gs_render_bwd's ordering reads; the rest is
 *     unused.  The orders change only the scheduling, never a result.
 *   - words GS_ORDER_WORDS(T) onwards: the contribution bits.  For every
 *     sorted position k and every 8x8 quadrant q of k's tile (row-major:
 *     top-left, top-right, bottom-left, bottom-right), bit (k & 31) of word
 *     GS_ORDER_WORDS(T) + (k >> 5) * 4 + q is set when that Gaussian was
 *     blended into at least one pixel of the quadrant.  The call zeroes these
 *     words; there should be at least GS_MASK_WORDS(P, T) - GS_ORDER_WORDS(T)
 *     of them for P sorted pairs (positions beyond the buffer are not
 *     recorded, and the backward then visits them all: correct, slower).
 *   gs_render_bwd uses the bits to walk only the terms that contribute.
 */
/* Words of the dispatch-order block for an image of `n_tiles` tiles. */
#define GS_ORDER_WORDS(n_tiles) (12u * (unsigned)(n_tiles) + 256u)
/* Words of the optional contribution mask for `capacity` sorted pairs on an
   image of `n_tiles` tiles. */
#define GS_MASK_WORDS(capacity, n_tiles) (GS_ORDER_WORDS(n_tiles) + 4u * (((unsigned)(capacity) + 31u) / 32u))

GS_API int gs_render_fwd(const gs_camera* cam, const unsigned* ranges, const unsigned* ids, const float* mean2d,
                  const float* conic_opacity, const float* colors, float* image, float* final_T,
                  unsigned* n_contrib, unsigned* contrib_mask, unsigned mask_words, void* stream);

/*
 * gs_render_stats - work counts of gs_render_fwd, per pixel (the derived
 *   measures "evaluated" and "blended" terms; a diagnostic, not a stage of
 *   the method).  n_evaluated [H,W]: list entries the pixel evaluated before
 *   it stopped (the stopping entry included), or the tile's list length;
 *   n_blended [H,W]: terms composited.  Same inputs and decisions as
 *   gs_render_fwd.
 */
GS_API int gs_render_stats(const gs_camera* cam, const unsigned* ranges, const unsigned* ids, const float* mean2d,
                           const float* conic_opacity, unsigned* n_evaluated, unsigned* n_blended, void* stream);

/*
 * gs_render_bwd - reverse per-pixel traversal ([CB] 2, 3).  From T = final_T
 *   and the colour behind S = bg, for list positions n_contrib-1 down to 0
 *   (the terms the forward blended): T <- T / (1 - alpha);
 *   dL/dcolor += alpha T dL/dC; dL/dalpha = T (color - S) . dL/dC;
 *   S <- alpha color + (1 - alpha) S; through alpha = opacity G (zero when
 *   the alpha_max cap is active) to dL/dopacity and dL/dG, then
 *   dL/d(a, b, c) = G dL/dG (-dx^2/2, -dx dy, -dy^2/2) and
 *   dL/d(u, v) = G dL/dG (a dx + b dy, b dx + c dy).
 * contrib_mask / mask_words: the forward's mask (see gs_render_fwd), or NULL
 *   to let the backward find the contributing terms itself (slower; same
 *   results up to the order of floating-point sums).  With the mask, the
 *   call first writes its dispatch order (words [4T, 8T) of the block) from
 *   the forward's per-quadrant counts, then dispatches one warp per quadrant
 *   in that order.
 * Outputs (OVERWRITTEN; the call zeroes them first): dL_dmean2d [N,2];
 *   dL_dconic_opacity [N,4] = (dL/da, dL/db, dL/dc, dL/dopacity);
 *   dL_dcolor [N,3].  Summation order across pixels is unspecified
 *   (floating-point atomics), so results are not bit-reproducible.
 */
GS_API int gs_render_bwd(const gs_camera* cam, int N, const unsigned* ranges, const unsigned* ids,
                  const float* mean2d, const float* conic_opacity, const float* colors,
                  const float* final_T, const unsigned* n_contrib, const unsigned* contrib_mask,
                  unsigned mask_words, const float* dL_dimage, float* dL_dmean2d, float* dL_dconic_opacity,
                  float* dL_dcolor, void* stream);

/*
 * gs_preprocess_bwd - 2D gradients to 3D parameters by the chain rule
 *   ([CB] 4; [TR] D.4): the conic gradient through the 2x2 inverse,
 *   Sigma2 = V V^T with V = J R L and L = R_q diag(s); the perspective
 *   Jacobian's dependence on the camera-space mean; the projected mean;
 *   the quaternion normalisation.  Opacity and colour gradients pass through.
 * Inputs: the forward's parameters, radius and conic_opacity, and the
 *   outputs of gs_render_bwd.
 * Outputs are ACCUMULATED (+=) so that several cameras can sum into one set:
 *   dL_dmeans [N,3], dL_dscales [N,3], dL_dquats [N,4], dL_dopacity [N],
 *   dL_dcolors [N,3].  Culled Gaussians (radius 0) are left untouched.
 * grad2d_accum [N] / vis_count [N] (optional, both or neither; may be NULL):
 *   densification statistics ([TR] D.1: the position gradient of each
 *   Gaussian accumulated over the views): for every Gaussian visible in this
 *   view, grad2d_accum += |dL/dmean2d| (Euclidean norm, pixels) and
 *   vis_count += 1.  Their ratio is the mean view-space gradient norm.
 */
GS_API int gs_preprocess_bwd(const gs_camera* cam, int N, const float* means, const float* scales,
                      const float* quats, const int* radius, const float* conic_opacity,
                      const float* dL_dmean2d, const float* dL_dconic_opacity, const float* dL_dcolor2d,
                      float* dL_dmeans, float* dL_dscales, float* dL_dquats, float* dL_dopacity,
                      float* dL_dcolors, float* grad2d_accum, unsigned* vis_count, void* stream);

/*
 * gs_sh_fwd / gs_sh_bwd - colour from real spherical harmonics ([CB] 4: the
 *   colour gradient reaches the SH coefficients through the derivative of
 *   the SH basis, band-limited).  Orthonormal real SH of degree <= 3 in
 *   Cartesian form on d = normalise(mean - camera centre), camera centre =
 *   -R^T t; coefficients ordered k = l^2 + l + m (Y_00; Y_1-1 ~ y, Y_10 ~ z,
 *   Y_11 ~ x; ...).  colour = max(0, sum_{k < (degree+1)^2} Y_k(d) sh[k] +
 *   offset) per channel.
 * sh [N, K, 3] with (degree + 1)^2 <= K <= 16 coefficients stored per
 *   Gaussian (only the first (degree + 1)^2 are used); colors [N, 3]
 *   (written).
 * gs_sh_bwd ACCUMULATES (+=) into dL_dsh [N, K, 3] (first (degree+1)^2 rows)
 *   and into dL_dmeans [N, 3] (the view-direction path; add the geometric
 *   path with gs_preprocess_bwd).  Where the clamp is active the channel
 *   passes no gradient.
 */
#define GS_SH_MAX_DEGREE 3
GS_API int gs_sh_fwd(const gs_camera* cam, int N, int degree, int K, const float* means, const float* sh,
                     float offset, float* colors, void* stream);
GS_API int gs_sh_bwd(const gs_camera* cam, int N, int degree, int K, const float* means, const float* sh,
                     float offset, const float* dL_dcolors, float* dL_dsh, float* dL_dmeans, void* stream);

/*
 * gs_sh_fwd_f16 / gs_sh_bwd_f16 - the same two operations with the
 *   coefficients stored in half precision ([CB] 5 and 7 list half-precision
 *   storage as a memory optimisation): sh [N, K, 3] holds IEEE binary16 bit
 *   patterns (2-byte aligned), widened to fp32 on load; all arithmetic,
 *   colors, dL_dcolors, the accumulated dL_dsh [N, K, 3] and dL_dmeans stay
 *   fp32.  Results equal the fp32 entry points applied to the widened
 *   coefficients.  Same ownership, accumulation and error behaviour as above.
 */
GS_API int gs_sh_fwd_f16(const gs_camera* cam, int N, int degree, int K, const float* means,
                         const unsigned short* sh, float offset, float* colors, void* stream);
GS_API int gs_sh_bwd_f16(const gs_camera* cam, int N, int degree, int K, const float* means,
                         const unsigned short* sh, float offset, const float* dL_dcolors, float* dL_dsh,
                         float* dL_dmeans, void* stream);

/*
 * gs_adam_step - fused optimiser step for the Gaussians' parameters
 *   ([TR] C.2: Adam with one learning rate per parameter group and a linear
 *   warm-up of the position and scale rates; Adam after Kingma and Ba).
 *   Raw parameters: means [N,3], log_scales [N,3] (scales = exp), quats [N,4]
 *   (16-byte aligned; renormalised to unit length after the update),
 *   logit_opacity [N] (opacity = sigmoid), colors [N,C] (C = 3 for RGB,
 *   3 * K for K spherical-harmonics coefficients; C = 0 skips the group).
 *   Gradients are those the rasterizer returns, w.r.t. the ACTIVATED values
 *   (dL_dscales w.r.t. exp(log_scales), dL_dopacity w.r.t. the opacity); they
 *   are chained through exp / sigmoid here.  step counts from 1; the rate of
 *   means and log_scales is multiplied by min(1, step / warmup_steps)
 *   (warmup_steps = 0: no warm-up).
 * m, v [(11 + C) N] each: first and second moments, group-major layout
 *   [means 3N | log_scales 3N | quats 4N | opacity N | colors C N]; zero them
 *   before step 1.  Parameters, m and v are updated in place.
 * scales [N,3], opacity [N] (optional, NULL to skip): written with the new
 *   activated values, ready for gs_preprocess_fwd.
 * Errors: GS_ERR_INVALID_ARG for step < 1, negative sizes, betas outside
 *   [0, 1), negative eps, missing pointers or unaligned quaternions.
 */
typedef struct {
    float lr_means, lr_scales, lr_quats, lr_opacity, lr_colors;
    float beta1, beta2, eps;
    int warmup_steps;
} gs_adam_config;

GS_API int gs_adam_step(const gs_adam_config* cfg, int step, int N, int C, float* means, float* log_scales,
                        float* quats, float* logit_opacity, float* colors, const float* dL_dmeans,
                        const float* dL_dscales, const float* dL_dquats, const float* dL_dopacity,
                        const float* dL_dcolors, float* m, float* v, float* scales, float* opacity, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GS_H */
