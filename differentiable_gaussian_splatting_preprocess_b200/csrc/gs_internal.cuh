// Internal helpers shared by the rasterizer's CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <set>
#include <utility>

#include "gs.h"

namespace gs {

constexpr int kTile = GS_TILE;
constexpr int kTilePixels = kTile * kTile;  // 256 pixels, one CTA per tile

// Workspace header at offset 0 of every workspace.  `status` collects
// device-detected error flags (sticky until gs_clear_status); `ticket` is the
// last-block counter of gs_preprocess_fwd and returns to 0 after each call.
struct WsHeader {
    unsigned status;
    unsigned ticket;
    unsigned reserved[62];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Host-side count of the kernels this library has launched (gs_launch_count);
// called after every launch statement.
void note_launch();

// Kernels that use more than the default 48 KiB of dynamic shared memory
// must opt in once per device.  Done on first use and remembered, so later
// calls (including calls recorded into a CUDA graph) issue no attribute call.
template <typename Kernel>
void opt_in_smem(Kernel kernel, size_t bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void*>> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    if (done.insert({dev, reinterpret_cast<const void*>(kernel)}).second)
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

inline int tiles_x(const gs_camera& c) { return (c.width + kTile - 1) / kTile; }
inline int tiles_y(const gs_camera& c) { return (c.height + kTile - 1) / kTile; }

// Host-side validation of the camera record.
inline bool camera_ok(const gs_camera* c) {
    if (!c) return false;
    if (c->tile != kTile) return false;
    if (c->width < 1 || c->height < 1 || c->width > 65536 || c->height > 65536) return false;
    return true;
}

__host__ __device__ inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define GS_LAUNCH_CHECK()                                          \
    do {                                                           \
        if (cudaPeekAtLastError() != cudaSuccess) {                \
            (void)cudaGetLastError();                              \
            return GS_ERR_CUDA;                                    \
        }                                                          \
    } while (0)

__device__ __forceinline__ void raise_status(WsHeader* h, unsigned flag) { atomicOr(&h->status, flag); }

// Index checks of the debug build (GS_DEBUG, compiled with relocatable
// device code so that every translation unit shares g_debug).  Each returns
// whether the index is inside its limit; a failed check ORs GS_ERR_INDEX
// into the debug word, and the caller skips the access.  In the release
// build they are constant true and cost nothing.
#ifdef GS_DEBUG
struct DebugState {
    unsigned n_gauss;   // Gaussian ids must be below this
    unsigned capacity;  // sorted-list positions must be below this
    unsigned flags;     // GS_ERR_INDEX once a check failed
    unsigned pad;
};
extern __device__ DebugState g_debug;
__device__ __forceinline__ bool debug_check(bool ok) {
    if (!ok) atomicOr(&g_debug.flags, (unsigned)GS_ERR_INDEX);
    return ok;
}
__device__ __forceinline__ bool id_ok(unsigned j) { return debug_check(j < g_debug.n_gauss); }
__device__ __forceinline__ bool pos_ok(unsigned k) { return debug_check(k < g_debug.capacity); }
__device__ __forceinline__ bool end_ok(unsigned k) { return debug_check(k <= g_debug.capacity); }
#else
__device__ __forceinline__ constexpr bool id_ok(unsigned) { return true; }
__device__ __forceinline__ constexpr bool pos_ok(unsigned) { return true; }
__device__ __forceinline__ constexpr bool end_ok(unsigned) { return true; }
#endif

// exp(x) in fp32 as a fixed sequence of IEEE operations, so that any IEEE
// machine with a correctly rounded fused multiply-add reproduces every bit
// (the library's expf does not promise that, and a one-ulp difference can
// flip an alpha_min or T_min decision).  x is clamped to >= -87 (exp(-87) is
// still a normal float); x log2(e) = n + f with n = rint(x log2(e)) taken
// with the 1.5 * 2^23 shifter and |f| <= 1/2, f computed with log2(e) split
// into a high and a low part (argument reduction after Cody and Waite); 2^f = exp(f ln 2) is the degree-7 Taylor polynomial
// sum_k (ln 2)^k f^k / k! by Horner's rule with fused multiply-adds
// (truncation below 6e-9 relative); n is added to the result's exponent bits.
#define GS_EXP_LOG2E 0x1.715476p+0f
#define GS_EXP_LOG2E_LO 0x1.4ae0c0p-26f
#define GS_EXP_SHIFT 0x1.8p+23f
#define GS_EXP_C7 0x1.ffcbfcp-17f
#define GS_EXP_C6 0x1.430912p-13f
#define GS_EXP_C5 0x1.5d87fep-10f
#define GS_EXP_C4 0x1.3b2ab6p-7f
#define GS_EXP_C3 0x1.c6b08ep-5f
#define GS_EXP_C2 0x1.ebfbe0p-3f
#define GS_EXP_C1 0x1.62e430p-1f

__device__ __forceinline__ float2 exp_pair(float2 x) {
    x = make_float2(fmaxf(x.x, -87.0f), fmaxf(x.y, -87.0f));
    const float2 l2e = make_float2(GS_EXP_LOG2E, GS_EXP_LOG2E);
    const float2 t = __ffma2_rn(x, l2e, make_float2(GS_EXP_SHIFT, GS_EXP_SHIFT));
    const float2 n = __fadd2_rn(t, make_float2(-GS_EXP_SHIFT, -GS_EXP_SHIFT));
    float2 f = __ffma2_rn(x, l2e, make_float2(-n.x, -n.y));
    f = __ffma2_rn(x, make_float2(GS_EXP_LOG2E_LO, GS_EXP_LOG2E_LO), f);
    float2 p = make_float2(GS_EXP_C7, GS_EXP_C7);
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C6, GS_EXP_C6));
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C5, GS_EXP_C5));
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C4, GS_EXP_C4));
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C3, GS_EXP_C3));
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C2, GS_EXP_C2));
    p = __ffma2_rn(p, f, make_float2(GS_EXP_C1, GS_EXP_C1));
    p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
    const unsigned sb = __float_as_uint(GS_EXP_SHIFT);
    const unsigned e0 = __float_as_uint(t.x) - sb, e1 = __float_as_uint(t.y) - sb;
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (e0 << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (e1 << 23)));
}

// One (pixel, Gaussian) term of the compositing sum, for two pixels of one
// row (px.x, px.y share py), with packed fp32x2 operations:
//   d = p - mean; power = -1/2 d^T A d = -1/2 (a dx^2 + 2 b dx dy + c dy^2);
//   alpha = min(alpha_max, opacity exp(power)).
// Every operation is an explicit round-to-nearest one in a fixed order (each
// lane of a packed operation rounds like the scalar one), so the forward and
// the backward kernels take bit-identical skip decisions and alphas, and an
// IEEE fp32 implementation of the same steps reproduces them.
// ok0 / ok1 are false when the term is skipped (power > 0 or alpha < alpha_min).
struct TermPair {
    float2 dx, G, at, alpha;
    float dy;
    bool ok0, ok1;
};

__device__ __forceinline__ void eval_pair(float2 px, float py, float2 xy, float4 co, float alpha_max,
                                          float alpha_min, TermPair& e) {
    e.dx = __fadd2_rn(px, make_float2(-xy.x, -xy.x));
    e.dy = __fsub_rn(py, xy.y);
    // q = a dx^2 + 2 b dx dy + c dy^2 with explicit fused multiply-adds: no
    // product feeds an addition, so the compiler has no contraction left to
    // choose (it does fuse packed multiplies into following packed adds).
    const float qc = __fmul_rn(__fmul_rn(co.z, e.dy), e.dy);
    const float2 adx = __fmul2_rn(make_float2(co.x, co.x), e.dx);
    const float2 bdx2 = __fmul2_rn(make_float2(2.0f * co.y, 2.0f * co.y), e.dx);
    float2 q = __ffma2_rn(adx, e.dx, make_float2(qc, qc));
    q = __ffma2_rn(bdx2, make_float2(e.dy, e.dy), q);
    const float2 power = __fmul2_rn(make_float2(-0.5f, -0.5f), q);
    e.G = exp_pair(power);
    e.at = __fmul2_rn(make_float2(co.w, co.w), e.G);
    e.alpha = make_float2(fminf(alpha_max, e.at.x), fminf(alpha_max, e.at.y));
    e.ok0 = !(power.x > 0.0f) && !(e.alpha.x < alpha_min);
    e.ok1 = !(power.y > 0.0f) && !(e.alpha.y < alpha_min);
}

// Culling parameters of one Gaussian, computed once per staged Gaussian:
//  - thr: a pixel can reach alpha >= alpha_min only where q = d^T A d <= thr.
//    The region is the ellipse q <= 2 ln(opacity / alpha_min); thr inflates
//    that bound to cover the fp32 rounding of `power` in eval_pair, whose
//    error grows with the conic's condition number (bounded by
//    (a + c)^2 / det), and of exp.  +inf when no bound is available (never
//    culled), -1 when the Gaussian can never reach alpha_min;
//  - box: the axis-aligned box (pixel coordinates xmin, xmax, ymin, ymax) of
//    that inflated ellipse, with extents sqrt(thr (A^-1)_xx) and
//    sqrt(thr (A^-1)_yy); a warp whose pixels all lie outside may skip the
//    Gaussian without changing any result.  A non-finite or undefined bound
//    gives the infinite box (never skipped);
//  - boc = b / c and boa = b / a, used by ellipse_misses.
struct CullParams {
    float4 box;
    float thr, boc, boa;
};

// The parameters use the hardware's approximate reciprocal, logarithm and
// reciprocal square root (a few ulp, a log error below 5e-7 absolute): the
// margins above (x1.001 and +1e-5 on thr, +0.01 px on the box, the minimiser
// of ellipse_misses only moving q upwards quadratically) dwarf those errors,
// and a result that is not finite leaves the Gaussian unculled.
__device__ __forceinline__ float sqrt_approx(float x) { return x > 0.0f ? x * rsqrtf(x) : 0.0f; }

__device__ __forceinline__ CullParams cull_params(float2 xy, float4 co, float alpha_min) {
    const float inf = __int_as_float(0x7f800000);
    CullParams cp;
    cp.box = make_float4(-inf, inf, -inf, inf);
    cp.thr = inf;
    cp.boc = __fdividef(co.y, co.z);
    cp.boa = __fdividef(co.y, co.x);
    if (!(alpha_min > 0.0f)) return cp;
    if (co.w < alpha_min) {  // alpha <= opacity < alpha_min
        cp.box = make_float4(inf, -inf, inf, -inf);
        cp.thr = -1.0f;
        return cp;
    }
    const float det = co.x * co.z - co.y * co.y;
    if (!(det > 0.0f)) return cp;
    const float tr = co.x + co.z;
    const float rdet = __fdividef(1.0f, det);
    const float ki = 2.0f * __logf(__fdividef(co.w, alpha_min)) * (1.001f + 1e-6f * (tr * tr * rdet)) + 1e-5f;
    if (!isfinite(ki)) return cp;
    cp.thr = ki;
    const float ex = sqrt_approx(ki * co.z * rdet) + 0.01f;
    const float ey = sqrt_approx(ki * co.x * rdet) + 0.01f;
    const float4 b = make_float4(xy.x - ex, xy.x + ex, xy.y - ey, xy.y + ey);
    if (isfinite(b.x) && isfinite(b.y) && isfinite(b.z) && isfinite(b.w)) cp.box = b;
    return cp;
}

// True when q = a dx^2 + 2 b dx dy + c dy^2 exceeds `thr` at every point of
// the rectangle [x0, x1] x [y0, y1] around the Gaussian's mean xy, i.e. when
// no pixel centre inside can reach alpha >= alpha_min.  The minimum of the
// positive-definite q over the rectangle is 0 when the mean is inside, else
// it lies on an edge, where q is a quadratic in one variable minimised in
// closed form (boc = b / c, boa = b / a) and clamped to the edge.  Any
// undefined value keeps the Gaussian (the comparison is false).
__device__ __forceinline__ bool ellipse_misses(float2 xy, float4 co, float thr, float boc, float boa, float x0,
                                               float x1, float y0, float y1) {
    if (xy.x >= x0 && xy.x <= x1 && xy.y >= y0 && xy.y <= y1) return false;
    const float a = co.x, b = co.y, c = co.z;
    if (!(a > 0.0f && c > 0.0f)) return false;
    const float ex0 = x0 - xy.x, ex1 = x1 - xy.x, ey0 = y0 - xy.y, ey1 = y1 - xy.y;
    float best = __int_as_float(0x7f800000);
    // edges x = x0 and x = x1: minimise over dy in [ey0, ey1]; dy* = -b dx / c
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const float dx = e ? ex1 : ex0;
        const float dy = fminf(fmaxf(-boc * dx, ey0), ey1);
        best = fminf(best, a * dx * dx + 2.0f * b * dx * dy + c * dy * dy);
    }
    // edges y = y0 and y = y1: minimise over dx in [ex0, ex1]; dx* = -b dy / a
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const float dy = e ? ey1 : ey0;
        const float dx = fminf(fmaxf(-boa * dy, ex0), ex1);
        best = fminf(best, a * dx * dx + 2.0f * b * dx * dy + c * dy * dy);
    }
    return best > thr;
}

// True when the box misses the rectangle of pixel centres [x0, x1] x [y0, y1].
__device__ __forceinline__ bool box_misses(float4 b, float x0, float x1, float y0, float y1) {
    return b.y < x0 || b.x > x1 || b.w < y0 || b.z > y1;
}

}  // namespace gs
