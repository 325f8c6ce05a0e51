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
// Per-Gaussian partial gradients are reduced across the warp before any
// global atomic: with the forward's contribution mask, one 9-lane atomic
// instruction per (quadrant, Gaussian); without it, the warps' sums are
// added in shared memory first and a (tile, Gaussian) pair costs one float2,
// one float4 and three float atomics.

#include <cuda_runtime.h>

#include "gs_internal.cuh"
#include "pdl.cuh"

namespace gs {
namespace {

// One CTA per 16x16 tile with 128 threads: each thread owns two horizontally
// adjacent pixels, evaluated together with packed fp32x2 arithmetic; warp w
// owns one 8x8 quadrant of the tile.  Gaussians are staged 128 at a time
// (the forward; 256 in the backward without the mask), each with its culling
// parameters computed once for the four warps.
// Before a warp walks a batch it builds a ballot mask of the staged
// Gaussians that can reach alpha >= alpha_min somewhere in its quadrant (a
// box test, then an exact ellipse-versus-rectangle test, both inflated for
// fp32 rounding) and walks only those: a skipped Gaussian would have been
// rejected by the alpha_min test at every pixel of the quadrant, so results
// are unchanged.
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 256;       // staged Gaussians per batch (backward without the mask)
constexpr int kWords = kBatch / 32;
constexpr int kFwdBatch = 128;    // staged Gaussians per batch of the forward
constexpr int kFwdWords = kFwdBatch / 32;
static_assert(kThreads * 2 == kTilePixels, "two pixels per thread");

struct PixelPair {
    int x0, y;
    bool in0, in1;
    float2 px;
    float py;
    float sx0, sx1, sy0, sy1;  // pixel-centre rectangle of this warp's quadrant
};

__device__ __forceinline__ PixelPair pixel_pair(const gs_camera& cam, int TX, int tile) {
    PixelPair q;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bx = (tile % TX) * kTile + (warp & 1) * 8;
    const int by = (tile / TX) * kTile + (warp >> 1) * 8;
    q.x0 = bx + 2 * (lane & 3);
    q.y = by + (lane >> 2);
    q.in0 = q.x0 < cam.width && q.y < cam.height;
    q.in1 = q.x0 + 1 < cam.width && q.y < cam.height;
    q.px = make_float2((float)q.x0 + 0.5f, (float)q.x0 + 1.5f);
    q.py = (float)q.y + 0.5f;
    q.sx0 = (float)bx + 0.5f;
    q.sx1 = q.sx0 + 7.0f;
    q.sy0 = (float)by + 0.5f;
    q.sy1 = q.sy0 + 7.0f;
    return q;
}

// The pixel pair of this lane in quadrant `quad` (0..3: 8x8 quarters of the
// tile, row-major) of tile `tile`.
__device__ __forceinline__ PixelPair quad_pixel_pair(const gs_camera& cam, int TX, int tile, int quad, int lane) {
    PixelPair q;
    const int bx = (tile % TX) * kTile + (quad & 1) * 8;
    const int by = (tile / TX) * kTile + (quad >> 1) * 8;
    q.x0 = bx + 2 * (lane & 3);
    q.y = by + (lane >> 2);
    q.in0 = q.x0 < cam.width && q.y < cam.height;
    q.in1 = q.x0 + 1 < cam.width && q.y < cam.height;
    q.px = make_float2((float)q.x0 + 0.5f, (float)q.x0 + 1.5f);
    q.py = (float)q.y + 0.5f;
    q.sx0 = (float)bx + 0.5f;
    q.sx1 = q.sx0 + 7.0f;
    q.sy0 = (float)by + 0.5f;
    q.sy1 = q.sy0 + 7.0f;
    return q;
}

// Can the staged Gaussian reach alpha >= alpha_min in this warp's quadrant?
// (box test, then the exact ellipse test; tr = (thr, b / c, b / a))
__device__ __forceinline__ bool may_contribute(float4 box, float4 tr, float2 xy, float4 co, const PixelPair& q) {
    if (box_misses(box, q.sx0, q.sx1, q.sy0, q.sy1)) return false;
    return !ellipse_misses(xy, co, tr.x, tr.y, tr.z, q.sx0, q.sx1, q.sy0, q.sy1);
}

// A tile's range of the sorted list; in the debug build, an empty range if it
// is not inside the list's capacity.
__device__ __forceinline__ uint2 checked_range(uint2 rg) {
    return (rg.x <= rg.y && end_ok(rg.y)) ? rg : make_uint2(0u, 0u);
}

// A staged entry that contributes nothing (zero opacity, never kept by the
// cull), used by the debug build in place of an entry whose index failed its
// check.
__device__ __forceinline__ void stage_inert(float2& xy, float4& co, float4& col, float4& box, float4& thr) {
    const float inf = __int_as_float(0x7f800000);
    xy = make_float2(0.0f, 0.0f);
    co = make_float4(1.0f, 0.0f, 1.0f, 0.0f);
    col = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    box = make_float4(inf, -inf, inf, -inf);
    thr = make_float4(-1.0f, 0.0f, 0.0f, 0.0f);
}

// Stage the culling parameters of one Gaussian (once per CTA and batch).
__device__ __forceinline__ void stage_cull(float2 xy, float4 co, float alpha_min, float4& box, float4& tr) {
    const CullParams cp = cull_params(xy, co, alpha_min);
    box = cp.box;
    tr = make_float4(cp.thr, cp.boc, cp.boa, 0.0f);
}

// Monotone 8-bit class of a work count, for the heaviest-first dispatch
// order (see order_by_work): exact below 16, then 8 classes per octave (at
// most 16 + 27 * 8 + 7 = 239).  Within a class the work differs by less than
// 1/8.
__device__ __forceinline__ unsigned order_code(unsigned w) {
    if (w < 16u) return w;
    const unsigned e = 31u - __clz(w);  // 4 .. 31
    return 16u + (e - 4u) * 8u + ((w >> (e - 3u)) & 7u);
}
constexpr int kOrderCodes = 256;
constexpr unsigned kPartUnits = 2048;  // quadrants per partition of the backward's order

__global__ void __launch_bounds__(kThreads)
k_render_fwd(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
             const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
             const float* __restrict__ colors, float* __restrict__ image, float* __restrict__ final_T,
             unsigned* __restrict__ n_contrib, unsigned* __restrict__ cmask, unsigned cmask_words,
             const unsigned* __restrict__ order, unsigned* __restrict__ quad_work,
             unsigned* __restrict__ part_hist) {
    pdl_enter();
    // two staging buffers: batch k is staged into buffer k & 1 while no warp
    // can still be reading it (its last readers processed batch k - 2 before
    // the barrier of batch k - 1), so one block barrier per batch suffices
    __shared__ float2 s_xy2[2][kFwdBatch];
    __shared__ float4 s_co2[2][kFwdBatch];
    __shared__ float4 s_col2[2][kFwdBatch];
    __shared__ float4 s_box2[2][kFwdBatch];
    __shared__ float4 s_thr2[2][kFwdBatch];  // threshold, b / c, b / a
    const unsigned tile = order ? order[blockIdx.x] : blockIdx.x;
    if (tile >= gridDim.x) return;  // not a permutation of the tiles: nothing valid to do
    const PixelPair q = pixel_pair(cam, TX, (int)tile);
    const int lane = threadIdx.x & 31;
    const uint2 rg = checked_range(ranges[tile]);
    const float amax = cam.alpha_max, amin = cam.alpha_min, tmin = cam.T_min;
    unsigned n_blend_pos = 0;  // list positions blended into some pixel of this warp

    float2 T = make_float2(1.0f, 1.0f);
    float2 C0 = make_float2(0.0f, 0.0f), C1 = C0, C2 = C0;
    unsigned last0 = 0, last1 = 0;
    bool done0 = !q.in0, done1 = !q.in1;
    static_assert(kFwdBatch == kThreads, "one staged entry per thread and batch");
    // each thread's list entry of the next batch is read one batch ahead, so
    // that staging a batch waits for one round of loads, not two
    unsigned j_next = (rg.x + threadIdx.x < rg.y && pos_ok(rg.x + threadIdx.x)) ? ids[rg.x + threadIdx.x] : 0xFFFFFFFFu;
    int buf = 0;
    for (unsigned b = rg.x; b < rg.y; b += kFwdBatch, buf ^= 1) {
        float2* const s_xy = s_xy2[buf];
        float4* const s_co = s_co2[buf];
        float4* const s_col = s_col2[buf];
        float4* const s_box = s_box2[buf];
        float4* const s_thr = s_thr2[buf];
        {
            const int r = threadIdx.x;
            const unsigned k = b + r;
            const unsigned j = j_next;
            const unsigned kn = k + kFwdBatch;
            j_next = (kn < rg.y && pos_ok(kn)) ? ids[kn] : 0xFFFFFFFFu;
            if (k < rg.y) {
                if (id_ok(j)) {
                    const float2 xy = mean2d[j];
                    const float4 co = conic_opacity[j];
                    s_xy[r] = xy;
                    s_co[r] = co;
                    s_col[r] = make_float4(colors[3 * j], colors[3 * j + 1], colors[3 * j + 2], 0.0f);
                    stage_cull(xy, co, amin, s_box[r], s_thr[r]);
                } else {  // debug build, failed check: an inert entry (zero opacity)
                    stage_inert(s_xy[r], s_co[r], s_col[r], s_box[r], s_thr[r]);
                }
            }
        }
        // the batch is staged; stop here if every pixel of the tile is done
        if (__syncthreads_count(done0 && done1) == kThreads) break;
        const int n = min((unsigned)kFwdBatch, rg.y - b);
        bool warp_done = __all_sync(0xffffffffu, done0 && done1);
        // cull against the pixels of this warp that are still compositing
        PixelPair qa = q;
        if (!warp_done) {
            const int ax0 = done0 ? 0x7fffffff : q.x0, ax1 = done1 ? -1 : q.x0 + 1;
            const int axmin = __reduce_min_sync(0xffffffffu, min(ax0, done1 ? 0x7fffffff : q.x0 + 1));
            const int axmax = __reduce_max_sync(0xffffffffu, max(ax1, done0 ? -1 : q.x0));
            const int ay = (done0 && done1) ? -1 : q.y;
            const int aymin = __reduce_min_sync(0xffffffffu, ay < 0 ? 0x7fffffff : ay);
            const int aymax = __reduce_max_sync(0xffffffffu, ay);
            qa.sx0 = (float)axmin + 0.5f;
            qa.sx1 = (float)axmax + 0.5f;
            qa.sy0 = (float)aymin + 0.5f;
            qa.sy1 = (float)aymax + 0.5f;
        }
        for (int w = 0; w < kFwdWords && !warp_done; ++w) {
            const int jl = w * 32 + lane;
            const bool keep = jl < n && may_contribute(s_box[jl], s_thr[jl], s_xy[jl], s_co[jl], qa);
            unsigned m = __ballot_sync(0xffffffffu, keep);
            unsigned blended_word = 0;  // bit l: staged Gaussian w*32+l blended some pixel of this warp
            while (m) {
                const int jj = w * 32 + __ffs(m) - 1;
                m &= m - 1;
                TermPair e;
                eval_pair(q.px, q.py, s_xy[jj], s_co[jj], amax, amin, e);
                const float2 Tn = __fmul2_rn(T, __fadd2_rn(make_float2(1.0f, 1.0f),
                                                           make_float2(-e.alpha.x, -e.alpha.y)));
                const bool use0 = !done0 && e.ok0, use1 = !done1 && e.ok1;
                const bool stop0 = use0 && Tn.x < tmin, stop1 = use1 && Tn.y < tmin;
                const bool blend0 = use0 && !stop0, blend1 = use1 && !stop1;
                done0 = done0 || stop0;
                done1 = done1 || stop1;
                const float2 wgt = make_float2(blend0 ? e.alpha.x * T.x : 0.0f, blend1 ? e.alpha.y * T.y : 0.0f);
                const float4 c = s_col[jj];
                C0 = __ffma2_rn(wgt, make_float2(c.x, c.x), C0);
                C1 = __ffma2_rn(wgt, make_float2(c.y, c.y), C1);
                C2 = __ffma2_rn(wgt, make_float2(c.z, c.z), C2);
                const unsigned pos = b - rg.x + (unsigned)jj + 1u;
                if (blend0) { T.x = Tn.x; last0 = pos; }
                if (blend1) { T.y = Tn.y; last1 = pos; }
                if (__any_sync(0xffffffffu, blend0 || blend1)) blended_word |= 1u << (jj & 31);
                if (__all_sync(0xffffffffu, done0 && done1)) {
                    warp_done = true;
                    break;
                }
            }
            n_blend_pos += __popc(blended_word);
            // record the word at global list positions b + w*32 .. b + w*32 + 31
            // (bit for position k: word (k >> 5) * 4 + warp, bit k & 31)
            if (cmask && blended_word && lane == 0) {
                const unsigned k0 = b + (unsigned)(w * 32);
                const unsigned o = k0 & 31u;
                const unsigned wi = (k0 >> 5) * kWarps + (threadIdx.x >> 5);
                if (wi < cmask_words) atomicOr(&cmask[wi], blended_word << o);
                if (o && wi + kWarps < cmask_words) atomicOr(&cmask[wi + kWarps], blended_word >> (32u - o));
            }
        }
    }
    // this quadrant's work for the backward's dispatch order: its count, and
    // one more of its class in its partition's histogram
    if (quad_work && lane == 0) {
        const unsigned u = 4u * tile + (threadIdx.x >> 5);
        quad_work[u] = n_blend_pos;
        atomicAdd(&part_hist[(u / kPartUnits) * kOrderCodes + order_code(n_blend_pos)], 1u);
    }
    const size_t plane = (size_t)cam.width * cam.height;
    const size_t pix = (size_t)q.y * cam.width + q.x0;
    if (q.in0) {
        image[pix] = fmaf(T.x, cam.bg[0], C0.x);
        image[plane + pix] = fmaf(T.x, cam.bg[1], C1.x);
        image[2 * plane + pix] = fmaf(T.x, cam.bg[2], C2.x);
        final_T[pix] = T.x;
        n_contrib[pix] = last0;
    }
    if (q.in1) {
        image[pix + 1] = fmaf(T.y, cam.bg[0], C0.y);
        image[plane + pix + 1] = fmaf(T.y, cam.bg[1], C1.y);
        image[2 * plane + pix + 1] = fmaf(T.y, cam.bg[2], C2.y);
        final_T[pix + 1] = T.y;
        n_contrib[pix + 1] = last1;
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

// One term of the reverse traversal for this thread's two pixels: undo the
// term's transmittance step, accumulate the colour behind it, and produce the
// pixel pair's share of the 9 gradient values (dL/du, dL/dv, dL/da, dL/db,
// dL/dc, dL/dr, dL/dg, dL/dopacity; dL/db_colour in r9).  p is the term's
// position in the tile's list; last0/last1 the pixels' contributor counts;
// terms the forward did not blend contribute nothing.  With kVote, returns
// false, with nothing changed, when no pixel of the warp takes the term (a
// warp vote; callers that only visit terms the forward blended in this warp
// skip it).  With kFold, dL/da, dL/db and dL/dc are left without their
// constant factors -1/2, -1 and -1/2 (exact powers of two, applied once after
// the warp sum).
// Sg = g . S, the upstream gradient dotted with the colour behind the term:
// dL/dalpha = T (g . c - Sg), and S <- alpha c + (1 - alpha) S becomes
// Sg <- Sg + alpha (g . c - Sg), one scalar per pixel instead of a colour.
template <bool kVote, bool kFold>
__device__ __forceinline__ bool bwd_term(const PixelPair& q, float2 xy, float4 co, float4 c, int p, unsigned last0,
                                         unsigned last1, float amax, float amin, float2 g0, float2 g1, float2 g2,
                                         float2& T, float2& Sg, float (&v)[8], float& r9) {
    TermPair e;
    eval_pair(q.px, q.py, xy, co, amax, amin, e);
    const bool c0 = p < (int)last0 && e.ok0;
    const bool c1 = p < (int)last1 && e.ok1;
    if (kVote && !__any_sync(0xffffffffu, c0 || c1)) return false;
    const float2 G = make_float2(c0 ? e.G.x : 0.0f, c1 ? e.G.y : 0.0f);
    const float2 al = make_float2(c0 ? e.alpha.x : 0.0f, c1 ? e.alpha.y : 0.0f);
    if (c0) T.x = __fdividef(T.x, 1.0f - al.x);
    if (c1) T.y = __fdividef(T.y, 1.0f - al.y);
    const float2 wgt = __fmul2_rn(al, T);
    float2 gc = __fmul2_rn(make_float2(c.x, c.x), g0);  // g . c
    gc = __ffma2_rn(make_float2(c.y, c.y), g1, gc);
    gc = __ffma2_rn(make_float2(c.z, c.z), g2, gc);
    const float2 diff = __fadd2_rn(gc, make_float2(-Sg.x, -Sg.y));
    const float2 dLda = __fmul2_rn(diff, T);
    // colour behind the next term towards the front, dotted with g
    Sg = __ffma2_rn(al, diff, Sg);
    // exact derivative of min(alpha_max, opacity G): zero while capped
    const float2 Gf = make_float2(e.at.x <= amax ? G.x : 0.0f, e.at.y <= amax ? G.y : 0.0f);
    const float2 dsig = __fmul2_rn(Gf, dLda);                    // dL/dopacity
    const float2 h = __fmul2_rn(dsig, make_float2(co.w, co.w));  // dL/dpower
    const float2 hdx = __fmul2_rn(h, e.dx);
    const float2 hdy = __fmul2_rn(h, make_float2(e.dy, e.dy));
    float2 t2;
    t2 = __ffma2_rn(make_float2(co.x, co.x), hdx, __fmul2_rn(make_float2(co.y, co.y), hdy));
    v[0] = t2.x + t2.y;  // dL/du
    t2 = __ffma2_rn(make_float2(co.y, co.y), hdx, __fmul2_rn(make_float2(co.z, co.z), hdy));
    v[1] = t2.x + t2.y;  // dL/dv
    t2 = __fmul2_rn(hdx, e.dx);
    v[2] = kFold ? t2.x + t2.y : -0.5f * (t2.x + t2.y);  // dL/da
    t2 = __fmul2_rn(hdx, make_float2(e.dy, e.dy));
    v[3] = kFold ? t2.x + t2.y : -(t2.x + t2.y);  // dL/db
    t2 = __fmul2_rn(hdy, make_float2(e.dy, e.dy));
    v[4] = kFold ? t2.x + t2.y : -0.5f * (t2.x + t2.y);  // dL/dc
    t2 = __fmul2_rn(wgt, g0);
    v[5] = t2.x + t2.y;  // dL/dcolor r
    t2 = __fmul2_rn(wgt, g1);
    v[6] = t2.x + t2.y;  // dL/dcolor g
    v[7] = dsig.x + dsig.y;  // dL/dopacity
    t2 = __fmul2_rn(wgt, g2);
    r9 = t2.x + t2.y;  // dL/dcolor b
    return true;
}

constexpr int kGradStride = 9;  // floats per staged Gaussian in shared memory

// With the forward's contribution mask (kMask) the warps walk the recorded
// positions and need no culling data: the staged boxes and thresholds are
// dropped, which brings shared memory and registers down to ten CTAs per SM.
template <bool kMask>
__global__ void __launch_bounds__(kThreads, kMask ? 10 : 8)
k_render_bwd(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
             const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
             const float* __restrict__ colors, const float* __restrict__ final_T,
             const unsigned* __restrict__ n_contrib, const unsigned* __restrict__ cmask, unsigned cmask_words,
             const float* __restrict__ dL_dimage, float2* __restrict__ dL_dmean2d,
             float4* __restrict__ dL_dconic_opacity, float* __restrict__ dL_dcolor) {
    __shared__ unsigned s_id[kBatch];
    __shared__ float2 s_xy[kBatch];
    __shared__ float4 s_co[kBatch];
    __shared__ float4 s_col[kBatch];
    __shared__ float4 s_box[kMask ? 1 : kBatch];
    __shared__ float4 s_thr[kMask ? 1 : kBatch];  // threshold, b / c, b / a
    __shared__ float s_grad[kBatch * kGradStride];
    __shared__ unsigned s_max[kWarps];

    const PixelPair q = pixel_pair(cam, TX, blockIdx.x);
    const int lane = threadIdx.x & 31;
    const uint2 rg = checked_range(ranges[blockIdx.x]);
    const float amax = cam.alpha_max, amin = cam.alpha_min;
    const size_t plane = (size_t)cam.width * cam.height;
    const size_t pix = (size_t)q.y * cam.width + q.x0;

    float2 T = make_float2(0.0f, 0.0f), g0 = T, g1 = T, g2 = T;
    unsigned last0 = 0, last1 = 0;
    if (q.in0) {
        T.x = final_T[pix];
        last0 = n_contrib[pix];
        g0.x = dL_dimage[pix];
        g1.x = dL_dimage[plane + pix];
        g2.x = dL_dimage[2 * plane + pix];
    }
    if (q.in1) {
        T.y = final_T[pix + 1];
        last1 = n_contrib[pix + 1];
        g0.y = dL_dimage[pix + 1];
        g1.y = dL_dimage[plane + pix + 1];
        g2.y = dL_dimage[2 * plane + pix + 1];
    }
    // g . bg: the colour behind the last term is the background
    float2 Sg = __fmul2_rn(make_float2(cam.bg[0], cam.bg[0]), g0);
    Sg = __ffma2_rn(make_float2(cam.bg[1], cam.bg[1]), g1, Sg);
    Sg = __ffma2_rn(make_float2(cam.bg[2], cam.bg[2]), g2, Sg);

    // furthest list position any pixel of the warp / of the tile blended
    const unsigned wlast = __reduce_max_sync(0xffffffffu, max(last0, last1));
    if (lane == 0) s_max[threadIdx.x >> 5] = wlast;
    for (int i = threadIdx.x; i < kBatch * kGradStride; i += kThreads) s_grad[i] = 0.0f;
    __syncthreads();
    unsigned max_last = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) max_last = max(max_last, s_max[w]);
    max_last = min(max_last, rg.y - rg.x);  // stay inside the tile's list

    const int warp = threadIdx.x >> 5;
    for (int top = (int)max_last; top > 0; top -= kBatch) {
        // the forward's contribution bits for this batch, loaded early so that
        // their latency overlaps the staging below
        unsigned mbits = 0;  // bit w: staged Gaussian w * 32 + lane blended a pixel of this warp
        if (kMask) {
#pragma unroll
            for (int w = 0; w < kWords; ++w) {
                const int p = top - 1 - (w * 32 + lane);
                if (p >= 0) {
                    const unsigned k = rg.x + (unsigned)p;
                    const unsigned wi = (k >> 5) * kWarps + warp;
                    const unsigned bit = wi >= cmask_words || ((cmask[wi] >> (k & 31u)) & 1u);
                    mbits |= bit << w;
                }
            }
        }
        // stage positions top-1, top-2, ... so that staged order is back to front
        for (int r = threadIdx.x; r < kBatch; r += kThreads) {
            const int pos = top - 1 - r;
            if (pos >= 0) {
                const unsigned j = pos_ok(rg.x + pos) ? ids[rg.x + pos] : 0xFFFFFFFFu;
                if (id_ok(j)) {
                    const float2 xy = mean2d[j];
                    const float4 co = conic_opacity[j];
                    s_id[r] = j;
                    s_xy[r] = xy;
                    s_co[r] = co;
                    s_col[r] = make_float4(colors[3 * j], colors[3 * j + 1], colors[3 * j + 2], 0.0f);
                    if (!kMask) stage_cull(xy, co, amin, s_box[r], s_thr[r]);
                } else {  // debug build, failed check: an inert entry (zero opacity, id 0)
                    s_id[r] = 0u;
                    float4 box, thr;
                    stage_inert(s_xy[r], s_co[r], s_col[r], box, thr);
                    if (!kMask) { s_box[r] = box; s_thr[r] = thr; }
                }
            }
        }
        __syncthreads();
        const int n = min(kBatch, top);
        for (int w = 0; w < kWords; ++w) {
            const int jl = w * 32 + lane;
            const int p = top - 1 - jl;
            bool keep = jl < n && p < (int)wlast;
            if (kMask) {
                keep = keep && ((mbits >> w) & 1u);
            } else {
                keep = keep && may_contribute(s_box[jl], s_thr[jl], s_xy[jl], s_co[jl], q);
            }
            unsigned m = __ballot_sync(0xffffffffu, keep);
            while (m) {
                const int jj = w * 32 + __ffs(m) - 1;
                m &= m - 1;
                const int p = top - 1 - jj;
                float v[8], r9;
                if (!bwd_term<true, false>(q, s_xy[jj], s_co[jj], s_col[jj], p, last0, last1, amax, amin, g0, g1, g2, T,
                                           Sg, v, r9))
                    continue;
                const float r8 = reduce8(v, lane);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) r9 += __shfl_xor_sync(0xffffffffu, r9, o);
                // lanes 4i hold value i (i < 8); lane 1 holds the ninth
                float* sg = s_grad + jj * kGradStride;
                if ((lane & 3) == 0) atomicAdd(sg + (lane >> 2), r8);
                if (lane == 1) atomicAdd(sg + 8, r9);
            }
        }
        __syncthreads();
        // flush this batch: one set of global atomics per (tile, Gaussian)
        for (int r = threadIdx.x; r < n; r += kThreads) {
            float* sg = s_grad + r * kGradStride;
            const float a0 = sg[0], a1 = sg[1], a2 = sg[2], a3 = sg[3], a4 = sg[4];
            const float a5 = sg[5], a6 = sg[6], a7 = sg[7], a8 = sg[8];
            const bool any = (a0 != 0.f) | (a1 != 0.f) | (a2 != 0.f) | (a3 != 0.f) | (a4 != 0.f) | (a5 != 0.f) |
                             (a6 != 0.f) | (a7 != 0.f) | (a8 != 0.f);
            if (any) {
                const unsigned j = s_id[r];
                atomicAdd(&dL_dmean2d[j], make_float2(a0, a1));
                atomicAdd(&dL_dconic_opacity[j], make_float4(a2, a3, a4, a7));
                atomicAdd(&dL_dcolor[3 * j + 0], a5);
                atomicAdd(&dL_dcolor[3 * j + 1], a6);
                atomicAdd(&dL_dcolor[3 * j + 2], a8);
#pragma unroll
                for (int i = 0; i < kGradStride; ++i) sg[i] = 0.0f;
            }
        }
        __syncthreads();
    }
}

// Backward driven by the forward's contribution mask: one CTA of one warp
// per 8x8 quadrant (block b takes unit order[b]: tile unit / 4, quadrant
// unit % 4, the units dispatched most blended first), so that a warp that
// finishes frees its slot at once for the next quadrant.  The warp walks the
// mask words of its quadrant from its last contributor towards the front;
// for each word the lanes whose bit is set load that list entry into the
// warp's shared-memory slots, and the warp then takes the set bits from the
// back.  Every visited term was blended by some pixel of the quadrant, so no
// vote is needed.  After the butterfly, the 9 gradient sums sit in 9
// different lanes (value i in lane 4i, the ninth in lane 1), which scale
// them by their constant factor and add them to the Gaussian's 2D gradients
// with one atomic instruction.
constexpr int kBwdWarpBlocksPerSM = 32;  // 64 registers per thread

__global__ void __launch_bounds__(32, kBwdWarpBlocksPerSM)
k_render_bwd_warp(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
                  const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
                  const float* __restrict__ colors, const float* __restrict__ final_T,
                  const unsigned* __restrict__ n_contrib, const unsigned* __restrict__ cmask, unsigned cmask_words,
                  const float* __restrict__ dL_dimage, float* __restrict__ dL_dmean2d,
                  float* __restrict__ dL_dconic_opacity, float* __restrict__ dL_dcolor,
                  const unsigned* __restrict__ order) {
    pdl_enter();
    __shared__ float2 s_xy[32];
    __shared__ float4 s_co[32];
    __shared__ float4 s_col[32];
    const int lane = threadIdx.x;
    const unsigned unit = order[blockIdx.x];
    if (unit >= gridDim.x) return;  // not a permutation of the quadrants: nothing valid to do
    const int tile = (int)(unit >> 2), quad = (int)(unit & 3u);
    const PixelPair q = quad_pixel_pair(cam, TX, tile, quad, lane);
    const uint2 rg = checked_range(ranges[tile]);
    const float amax = cam.alpha_max, amin = cam.alpha_min;
    const size_t plane = (size_t)cam.width * cam.height;
    const size_t pix = (size_t)q.y * cam.width + q.x0;

    float2 T = make_float2(0.0f, 0.0f), g0 = T, g1 = T, g2 = T;
    unsigned last0 = 0, last1 = 0;
    if (q.in0) {
        T.x = final_T[pix];
        last0 = n_contrib[pix];
        g0.x = dL_dimage[pix];
        g1.x = dL_dimage[plane + pix];
        g2.x = dL_dimage[2 * plane + pix];
    }
    if (q.in1) {
        T.y = final_T[pix + 1];
        last1 = n_contrib[pix + 1];
        g0.y = dL_dimage[pix + 1];
        g1.y = dL_dimage[plane + pix + 1];
        g2.y = dL_dimage[2 * plane + pix + 1];
    }
    // g . bg: the colour behind the last term is the background
    float2 Sg = __fmul2_rn(make_float2(cam.bg[0], cam.bg[0]), g0);
    Sg = __ffma2_rn(make_float2(cam.bg[1], cam.bg[1]), g1, Sg);
    Sg = __ffma2_rn(make_float2(cam.bg[2], cam.bg[2]), g2, Sg);
    // furthest list position any pixel of this warp blended (a count), kept
    // inside the tile's list
    const unsigned wlast = min(__reduce_max_sync(0xffffffffu, max(last0, last1)), rg.y - rg.x);
    if (wlast == 0) return;

    // where this lane's flush goes: value i of the butterfly in lane 4i, the
    // ninth (blue) in lane 1; each lane adds to one component of one array,
    // after the constant factor of its value (-1/2, -1, -1/2 for a, b, c)
    float* gbase = nullptr;
    unsigned gstride = 0;
    float post = 1.0f;
    if (lane == 0 || lane == 4) { gbase = dL_dmean2d + (lane >> 2); gstride = 2; }
    else if (lane == 8 || lane == 12 || lane == 16) {
        gbase = dL_dconic_opacity + ((lane >> 2) - 2); gstride = 4; post = lane == 12 ? -1.0f : -0.5f;
    }
    else if (lane == 28) { gbase = dL_dconic_opacity + 3; gstride = 4; }
    else if (lane == 20 || lane == 24) { gbase = dL_dcolor + ((lane >> 2) - 5); gstride = 3; }
    else if (lane == 1) { gbase = dL_dcolor + 2; gstride = 3; }

    const unsigned k_hi = rg.x + wlast - 1;  // last list entry to visit (global index)
    for (int wk = (int)(k_hi >> 5); wk >= (int)(rg.x >> 5); --wk) {
        const unsigned kb = (unsigned)wk << 5;
        const unsigned wi = (unsigned)wk * kWarps + (unsigned)quad;
        unsigned bits = wi < cmask_words ? cmask[wi] : 0xFFFFFFFFu;
        // entries of this word that belong to the tile's list up to k_hi
        const unsigned lo = rg.x > kb ? rg.x - kb : 0u;
        const unsigned hi = k_hi - kb;  // < 32 only in the first (highest) word
        if (hi < 31u) bits &= (2u << hi) - 1u;
        bits &= ~((1u << lo) - 1u);
        if (!bits) continue;
        if ((bits >> lane) & 1u) {
            const unsigned j = pos_ok(kb + lane) ? ids[kb + lane] : 0xFFFFFFFFu;
            // the id rides in the colour's unused fourth lane (as its bits)
            if (id_ok(j)) {
                s_xy[lane] = mean2d[j];
                s_co[lane] = conic_opacity[j];
                s_col[lane] = make_float4(colors[3 * j], colors[3 * j + 1], colors[3 * j + 2], __uint_as_float(j));
            } else {  // debug build, failed check: an inert entry (zero opacity, id 0)
                float4 box, thr;
                stage_inert(s_xy[lane], s_co[lane], s_col[lane], box, thr);
                s_col[lane].w = __uint_as_float(0u);
            }
        }
        __syncwarp();
        // terms from the back; the next term's staged entry is loaded before
        // the current one is evaluated
        int l = 31 - __clz(bits);
        float2 xy = s_xy[l];
        float4 co = s_co[l], col = s_col[l];
        while (true) {
            bits &= ~(1u << l);
            const int ln = bits ? 31 - __clz(bits) : l;
            const float2 xy_n = s_xy[ln];
            const float4 co_n = s_co[ln], col_n = s_col[ln];
            const int p = (int)(kb + (unsigned)l - rg.x);
            float v[8], r9;
            bwd_term<false, true>(q, xy, co, col, p, last0, last1, amax, amin, g0, g1, g2, T, Sg, v, r9);
            const float r8 = reduce8(v, lane);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r9 += __shfl_xor_sync(0xffffffffu, r9, o);
            const float val = (lane == 1 ? r9 : r8) * post;
            // (a zero sum is added too: testing for it costs more than the atomic)
            if (gbase) atomicAdd(gbase + (size_t)__float_as_uint(col.w) * gstride, val);
            if (!bits) break;
            l = ln;
            xy = xy_n;
            co = co_n;
            col = col_n;
        }
        __syncwarp();  // the next word reuses this warp's slots
    }
}

// Dispatch order of the render CTAs, heaviest first.  The hardware starts
// CTAs roughly in block-index order; a heavy tile that starts late (the
// heavy tiles of a scene sit where its Gaussians crowd, anywhere in the
// image) keeps its SM busy after the others have gone idle.  Dispatching in
// decreasing order of work (longest processing time first) leaves the
// light CTAs for the end.  The forward orders its tiles by list length (its
// work before early termination is not known in advance); the backward
// orders its quadrants by the number of list positions the forward blended
// in them, which is the number of terms the quadrant's warp will visit.
// The order changes which CTA runs when, never what a CTA computes.

constexpr int kOrderThreads = 1024;
constexpr int kOrderWarps = kOrderThreads / 32;
constexpr int kOrderCntStride = kOrderCodes + 1;  // per-warp row of class counters, padded
constexpr int kOrderStage = 32768;                // items whose class and position stay in shared memory

struct OrderSmem {
    unsigned cnt[kOrderWarps * kOrderCntStride];  // (warp, class) at warp * 257 + class
    unsigned wsum[kOrderWarps];
    unsigned out[kOrderStage];                    // positions 0 .. kOrderStage-1 of the order
    unsigned char code[kOrderStage];              // classes of items 0 .. kOrderStage-1
};

// Counting sort by one CTA of kOrderThreads threads: order[0 .. n) = the
// items 0 .. n-1 in decreasing class (within a class in no particular order:
// the order only decides which CTA starts when).
//   0. the whole CTA loads the items' work counts (coalesced, many loads in
//      flight) and keeps their classes in shared memory;
//   1. warp w owns a contiguous run of 32-item rows and counts its items per
//      class in its own row of counters (shared-memory atomics: lanes of one
//      class serialise only within one instruction);
//   2. an exclusive scan over the counters in (decreasing class, warp) order
//      turns each into the first position of its (class, warp) group;
//   3. each warp walks its rows again and takes positions with the same
//      atomics; positions are gathered in shared memory and written out in
//      order.
// Items past kOrderStage (images of more than 8192 tiles) take the same
// steps with their class recomputed from global memory and their position
// stored directly.
template <class Work>
__device__ void order_by_work(unsigned n, Work work, unsigned* __restrict__ order, OrderSmem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kOrderWarps * kOrderCntStride; i += kOrderThreads) sm.cnt[i] = 0u;
    const unsigned nc = min(n, (unsigned)kOrderStage);
#pragma unroll 8
    for (unsigned i = threadIdx.x; i < nc; i += kOrderThreads) sm.code[i] = (unsigned char)order_code(work(i));
    __syncthreads();
    const unsigned rows = (n + 31u) / 32u;
    const unsigned per_warp = (rows + kOrderWarps - 1) / kOrderWarps;
    const unsigned i0 = min(rows, (unsigned)warp * per_warp) * 32u + lane;
    const unsigned i1 = min(n, min(rows, (unsigned)warp * per_warp + per_warp) * 32u);
    unsigned* cnt = sm.cnt + warp * kOrderCntStride;
    auto code_of = [&](unsigned i) { return i < nc ? (unsigned)sm.code[i] : order_code(work(i)); };
    // 1. counts per (warp, class)
#pragma unroll 4
    for (unsigned i = i0; i < i1; i += 32u) atomicAdd(&cnt[code_of(i)], 1u);
    __syncthreads();
    // 2. exclusive scan; thread t takes flat entries 8t .. 8t+7, flat entry
    // f = (255 - class) * 32 + warp
    constexpr int per = kOrderCodes * kOrderWarps / kOrderThreads;
    unsigned v[per], sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        const unsigned f = threadIdx.x * per + k;
        v[k] = sm.cnt[(f & 31u) * kOrderCntStride + (kOrderCodes - 1 - (f >> 5))];
        sum += v[k];
    }
    unsigned incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sm.wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const unsigned t = sm.wsum[lane];
        unsigned ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        sm.wsum[lane] = ti - t;
    }
    __syncthreads();
    unsigned run = sm.wsum[warp] + incl - sum;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        const unsigned f = threadIdx.x * per + k;
        sm.cnt[(f & 31u) * kOrderCntStride + (kOrderCodes - 1 - (f >> 5))] = run;
        run += v[k];
    }
    __syncthreads();
    // 3. positions
#pragma unroll 4
    for (unsigned i = i0; i < i1; i += 32u) {
        const unsigned pos = atomicAdd(&cnt[code_of(i)], 1u);
        if (pos < (unsigned)kOrderStage) sm.out[pos] = i;
        else order[pos] = i;
    }
    __syncthreads();
    for (unsigned p = threadIdx.x; p < nc; p += kOrderThreads) order[p] = sm.out[p];
}

__device__ __forceinline__ void zero_words(unsigned* __restrict__ a, size_t n, size_t first, size_t stride) {
    for (size_t i = first; i < n; i += stride) a[i] = 0u;
}

// Before the forward: block 0 orders the tiles by list length into
// tile_order[T]; the other blocks zero the backward's partition histograms
// and the contribution bits (one range).  Launched with
// sizeof(OrderSmem) bytes of dynamic shared memory (every block gets them;
// one block uses them).
__global__ void __launch_bounds__(kOrderThreads, 1)
k_fwd_prep(int T, const uint2* __restrict__ ranges, unsigned* __restrict__ tile_order, unsigned* __restrict__ bits,
           size_t n_bits) {
    pdl_enter();
    if (blockIdx.x == 0) {
        extern __shared__ __align__(16) unsigned char order_smem[];
        order_by_work((unsigned)T, [&](unsigned t) { const uint2 r = ranges[t]; return r.y - r.x; }, tile_order,
                      *reinterpret_cast<OrderSmem*>(order_smem));
        return;
    }
    zero_words(bits, n_bits, (size_t)(blockIdx.x - 1) * kOrderThreads + threadIdx.x,
               (size_t)(gridDim.x - 1) * kOrderThreads);
}

// Before the backward: blocks 0 .. P-1 order the 4T quadrants by the
// forward's blended-position counts into quad_order[4T] (decreasing class);
// the other blocks zero the gradient outputs.  The forward counted every
// partition's quadrants per class (part_hist[p][c], partition p = quadrants
// p * kPartUnits ..), so block p knows where each class begins for its
// quadrants - after every quadrant of a higher class, and after those of its
// class in lower partitions - and places them with shared-memory atomics
// (within a class in no particular order).
__global__ void __launch_bounds__(kOrderThreads)
k_bwd_prep(int T, int P, const unsigned* __restrict__ quad_work, const unsigned* __restrict__ part_hist,
           unsigned* __restrict__ quad_order, float* __restrict__ a, size_t na, float* __restrict__ b, size_t nb,
           float* __restrict__ c, size_t nc) {
    pdl_enter();
    if ((int)blockIdx.x < P) {
        __shared__ unsigned s_cur[kOrderCodes];
        __shared__ unsigned s_w[kOrderCodes / 32];
        const int p = blockIdx.x, t = threadIdx.x, lane = t & 31;
        unsigned tot = 0, before = 0;
        if (t < kOrderCodes) {
            const int cls = kOrderCodes - 1 - t;  // thread t: classes in decreasing order
            for (int q = 0; q < P; ++q) {
                const unsigned h = part_hist[q * kOrderCodes + cls];
                tot += h;
                before += q < p ? h : 0u;
            }
        }
        // exclusive scan of the class totals in decreasing class order
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (t < kOrderCodes && lane == 31) s_w[t >> 5] = incl;
        __syncthreads();
        if (t < kOrderCodes) {
            unsigned above = incl - tot;
            for (int w = 0; w < (t >> 5); ++w) above += s_w[w];
            s_cur[kOrderCodes - 1 - t] = above + before;
        }
        __syncthreads();
        const unsigned n = 4u * (unsigned)T;
        const unsigned u1 = min(n, (unsigned)(p + 1) * kPartUnits);
        for (unsigned u = (unsigned)p * kPartUnits + t; u < u1; u += kOrderThreads)
            quad_order[atomicAdd(&s_cur[order_code(quad_work[u])], 1u)] = u;
        return;
    }
    const size_t first = (size_t)(blockIdx.x - P) * kOrderThreads + threadIdx.x;
    const size_t stride = (size_t)(gridDim.x - P) * kOrderThreads;
    zero_words(reinterpret_cast<unsigned*>(a), na, first, stride);
    zero_words(reinterpret_cast<unsigned*>(b), nb, first, stride);
    zero_words(reinterpret_cast<unsigned*>(c), nc, first, stride);
}

// Work counts of the forward, per pixel: list entries evaluated before the
// pixel stopped (the stopping entry included) and terms blended.  One thread
// per pixel walking its tile's list in order with the same term evaluation as
// the forward (pixel duplicated in both lanes), so the counts are those of the
// compositing above.  A diagnostic for measurement, not part of the hot path.
__global__ void __launch_bounds__(kTilePixels)
k_render_stats(gs_camera cam, int TX, const uint2* __restrict__ ranges, const unsigned* __restrict__ ids,
               const float2* __restrict__ mean2d, const float4* __restrict__ conic_opacity,
               unsigned* __restrict__ n_evaluated, unsigned* __restrict__ n_blended) {
    const int tile = blockIdx.x;
    const int x = (tile % TX) * kTile + (threadIdx.x & (kTile - 1));
    const int y = (tile / TX) * kTile + (threadIdx.x / kTile);
    if (x >= cam.width || y >= cam.height) return;
    const uint2 rg = checked_range(ranges[tile]);
    const float2 px = make_float2((float)x + 0.5f, (float)x + 0.5f);
    const float py = (float)y + 0.5f;
    float T = 1.0f;
    unsigned ev = 0, bl = 0;
    for (unsigned k = rg.x; k < rg.y; ++k) {
        const unsigned j = pos_ok(k) ? ids[k] : 0xFFFFFFFFu;
        if (!id_ok(j)) break;
        ++ev;
        TermPair e;
        eval_pair(px, py, mean2d[j], conic_opacity[j], cam.alpha_max, cam.alpha_min, e);
        if (!e.ok0) continue;
        const float Tn = __fmul_rn(T, __fsub_rn(1.0f, e.alpha.x));
        if (Tn < cam.T_min) break;
        T = Tn;
        ++bl;
    }
    const size_t pix = (size_t)y * cam.width + x;
    n_evaluated[pix] = ev;
    n_blended[pix] = bl;
}

__global__ void k_zero(float* __restrict__ a, size_t na, float* __restrict__ b, size_t nb, float* __restrict__ c,
                       size_t nc) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < na; i += stride) a[i] = 0.0f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += stride) b[i] = 0.0f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nc; i += stride) c[i] = 0.0f;
}

// The contribution-mask buffer: the dispatch-order block, then the bits.
struct MaskParts {
    unsigned* quad_work = nullptr;    // [4T] blended positions per quadrant (forward output)
    unsigned* quad_order = nullptr;   // [4T] backward dispatch order
    unsigned* tile_order = nullptr;   // [T] forward dispatch order
    unsigned* part_hist = nullptr;    // [P][256] quadrants per (partition, class) (forward output)
    unsigned* bits = nullptr;         // contribution bits
    unsigned bits_words = 0;
    unsigned prep_words = 0;          // words from part_hist to the end: zeroed before the forward
    int parts = 0;                    // P = ceil(4T / kPartUnits)
};

// Splits a caller's mask buffer; false if it is too small or not a multiple
// of 4 words.
bool mask_parts(unsigned* mask, unsigned mask_words, int T, MaskParts& m) {
    if (!mask) return true;
    const size_t order_words = 12 * (size_t)T + 256;  // GS_ORDER_WORDS
    if (mask_words % kWarps != 0 || (size_t)mask_words < order_words + kWarps) return false;
    m.parts = (int)((4 * (size_t)T + kPartUnits - 1) / kPartUnits);
    m.quad_work = mask;
    m.quad_order = mask + 4 * (size_t)T;
    m.tile_order = mask + 8 * (size_t)T;
    m.part_hist = mask + 9 * (size_t)T;  // P * 256 <= T / 2 + 256 words, inside the block
    m.bits = mask + order_words;
    m.bits_words = mask_words - (unsigned)order_words;
    m.prep_words = mask_words - 9 * (unsigned)T;
    return true;
}

// Blocks of a prep kernel: the ordering block plus enough to zero `words`
// words, at most one block per SM in all (each holds sizeof(OrderSmem)).
int prep_blocks(size_t words) {
    const size_t z = (words + kOrderThreads - 1) / kOrderThreads;
    return 1 + (int)(z < 147 ? z : 147);
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" int gs_render_fwd(const gs_camera* cam, const unsigned* ranges, const unsigned* ids, const float* mean2d,
                             const float* conic_opacity, const float* colors, float* image, float* final_T,
                             unsigned* n_contrib, unsigned* contrib_mask, unsigned mask_words, void* stream) {
    if (!camera_ok(cam) || !ranges || !image || !final_T || !n_contrib) return GS_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || (conic_opacity && !aligned(conic_opacity, 16)) || (mean2d && !aligned(mean2d, 8)))
        return GS_ERR_INVALID_ARG;
    const int TX = tiles_x(*cam), T = TX * tiles_y(*cam);
    MaskParts m;
    if (!mask_parts(contrib_mask, mask_words, T, m)) return GS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (contrib_mask) {
        opt_in_smem(k_fwd_prep, sizeof(OrderSmem));
        launch_pdl(k_fwd_prep, prep_blocks(m.prep_words), kOrderThreads, sizeof(OrderSmem), st, T,
                   reinterpret_cast<const uint2*>(ranges), m.tile_order, m.part_hist, m.prep_words);
        note_launch();
        GS_LAUNCH_CHECK();
    }
    launch_pdl(k_render_fwd, T, kThreads, 0, st, *cam, TX, reinterpret_cast<const uint2*>(ranges), ids,
               reinterpret_cast<const float2*>(mean2d), reinterpret_cast<const float4*>(conic_opacity), colors, image,
               final_T, n_contrib, m.bits, m.bits_words, m.tile_order, m.quad_work, m.part_hist);
    note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

extern "C" int gs_render_bwd(const gs_camera* cam, int N, const unsigned* ranges, const unsigned* ids,
                             const float* mean2d, const float* conic_opacity, const float* colors,
                             const float* final_T, const unsigned* n_contrib, const unsigned* contrib_mask,
                             unsigned mask_words, const float* dL_dimage, float* dL_dmean2d,
                             float* dL_dconic_opacity, float* dL_dcolor, void* stream) {
    if (!camera_ok(cam) || N < 0 || !ranges || !final_T || !n_contrib || !dL_dimage) return GS_ERR_INVALID_ARG;
    if (N > 0 && (!dL_dmean2d || !dL_dconic_opacity || !dL_dcolor)) return GS_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || (conic_opacity && !aligned(conic_opacity, 16)) || (mean2d && !aligned(mean2d, 8)) ||
        (dL_dmean2d && !aligned(dL_dmean2d, 8)) || (dL_dconic_opacity && !aligned(dL_dconic_opacity, 16)))
        return GS_ERR_INVALID_ARG;
    const int TX = tiles_x(*cam), T = TX * tiles_y(*cam);
    // the buffer is only read here, except for the backward's own dispatch order
    MaskParts m;
    if (!mask_parts(const_cast<unsigned*>(contrib_mask), mask_words, T, m)) return GS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t n = (size_t)N;
    if (contrib_mask) {
        const size_t z = (n * 4 + kOrderThreads - 1) / kOrderThreads;
        const int zb = (int)(z < 148 * 2 ? (z ? z : 1) : 148 * 2);
        launch_pdl(k_bwd_prep, m.parts + zb, kOrderThreads, 0, st, T, m.parts, m.quad_work, m.part_hist,
                   m.quad_order, dL_dmean2d, n * 2, dL_dconic_opacity, n * 4, dL_dcolor, n * 3);
        note_launch();
        GS_LAUNCH_CHECK();
        launch_pdl(k_render_bwd_warp, 4 * T, 32, 0, st, *cam, TX, reinterpret_cast<const uint2*>(ranges), ids,
                   reinterpret_cast<const float2*>(mean2d), reinterpret_cast<const float4*>(conic_opacity), colors,
                   final_T, n_contrib, m.bits, m.bits_words, dL_dimage, dL_dmean2d, dL_dconic_opacity, dL_dcolor,
                   m.quad_order);
        note_launch();
        GS_LAUNCH_CHECK();
        return GS_OK;
    }
    if (N > 0) {
        int blocks = (int)((n * 4 + 255) / 256);
        if (blocks > 148 * 8) blocks = 148 * 8;
        k_zero<<<blocks, 256, 0, st>>>(dL_dmean2d, n * 2, dL_dconic_opacity, n * 4, dL_dcolor, n * 3); note_launch();
        GS_LAUNCH_CHECK();
    }
    auto kernel = k_render_bwd<false>;
    kernel<<<T, kThreads, 0, st>>>(*cam, TX, reinterpret_cast<const uint2*>(ranges), ids,
                                   reinterpret_cast<const float2*>(mean2d),
                                   reinterpret_cast<const float4*>(conic_opacity), colors, final_T, n_contrib,
                                   nullptr, 0u, dL_dimage, reinterpret_cast<float2*>(dL_dmean2d),
                                   reinterpret_cast<float4*>(dL_dconic_opacity), dL_dcolor); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}

extern "C" int gs_render_stats(const gs_camera* cam, const unsigned* ranges, const unsigned* ids, const float* mean2d,
                               const float* conic_opacity, unsigned* n_evaluated, unsigned* n_blended, void* stream) {
    if (!camera_ok(cam) || !ranges || !n_evaluated || !n_blended) return GS_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || (conic_opacity && !aligned(conic_opacity, 16)) || (mean2d && !aligned(mean2d, 8)))
        return GS_ERR_INVALID_ARG;
    const int TX = tiles_x(*cam), T = TX * tiles_y(*cam);
    k_render_stats<<<T, kTilePixels, 0, (cudaStream_t)stream>>>(
        *cam, TX, reinterpret_cast<const uint2*>(ranges), ids, reinterpret_cast<const float2*>(mean2d),
        reinterpret_cast<const float4*>(conic_opacity), n_evaluated, n_blended); note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}
