// Internal helpers shared by the rasterizer's CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

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

inline int tiles_x(const gs_camera& c) { return (c.width + kTile - 1) / kTile; }
inline int tiles_y(const gs_camera& c) { return (c.height + kTile - 1) / kTile; }

// Host-side validation of the camera record.
inline bool camera_ok(const gs_camera* c) {
    if (!c) return false;
    if (c->tile != kTile) return false;
    if (c->width < 1 || c->height < 1 || c->width > 65536 || c->height > 65536) return false;
    return true;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define GS_LAUNCH_CHECK()                                          \
    do {                                                           \
        if (cudaPeekAtLastError() != cudaSuccess) {                \
            (void)cudaGetLastError();                              \
            return GS_ERR_CUDA;                                    \
        }                                                          \
    } while (0)

__device__ __forceinline__ void raise_status(WsHeader* h, unsigned flag) { atomicOr(&h->status, flag); }

// One (pixel, Gaussian) term of the compositing sum.  Every operation is an
// explicit round-to-nearest intrinsic so that the forward and the backward
// kernels, compiled separately, take bit-identical skip decisions and alphas.
//   d = p - mean; power = -1/2 (a dx^2 + c dy^2) - b dx dy;
//   alpha = min(alpha_max, opacity exp(power)).
// Returns false when the term is skipped (power > 0 or alpha < alpha_min).
struct Term {
    float dx, dy, G, at, alpha;
};

__device__ __forceinline__ bool eval_term(float px, float py, float2 xy, float4 co, float alpha_max,
                                          float alpha_min, Term& e) {
    e.dx = __fsub_rn(px, xy.x);
    e.dy = __fsub_rn(py, xy.y);
    const float qa = __fmul_rn(__fmul_rn(co.x, e.dx), e.dx);
    const float qc = __fmul_rn(__fmul_rn(co.z, e.dy), e.dy);
    const float qb = __fmul_rn(__fmul_rn(co.y, e.dx), e.dy);
    const float power = __fsub_rn(__fmul_rn(-0.5f, __fadd_rn(qa, qc)), qb);
    if (power > 0.0f) return false;
    e.G = expf(power);
    e.at = __fmul_rn(co.w, e.G);
    e.alpha = fminf(alpha_max, e.at);
    return !(e.alpha < alpha_min);
}

}  // namespace gs
