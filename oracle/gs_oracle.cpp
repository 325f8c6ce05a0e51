// CPU oracle for the tile-based differentiable 3D Gaussian Splatting rasterizer.
//
// TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
// baseline leg of the benchmark may load this library.  The product path
// (the CUDA library and its Python binding) never calls it and shares no
// code, header, table or constant generator with it.
//
// What it computes is the plain definition of each stage, written out in the
// order the formulas are stated, with no blocking, fusion or reordering:
//
//   preprocess  Sigma3 = R S S^T R^T from a unit quaternion and scales
//               ("3DGS training and optimisation" page, section D.4 and the
//               CUDA-backward page, section 4); t = W mu + t_v; EWA projection
//               Sigma2 = (J W) Sigma3 (J W)^T + eps I; conic = Sigma2^-1;
//               radius = ceil(3 sqrt(lambda_max)); tile rectangle (the
//               training page, section E.3: AABB coarse cull per tile).
//   binning     every (tile, Gaussian) pair, sorted by (tile, depth, id)
//               (training page, section E.3: per-tile depth sort).
//   render fwd  front-to-back compositing C = sum_i c_i a_i prod_{j<i}(1 - a_j)
//               (backprop chain-rule page, rendering equation) with
//               a_i = min(0.99, sigma_i G_i), G_i = exp(-1/2 d^T A d)
//               (CUDA-backward page, section 2).
//   render bwd  the gradient table of the CUDA-backward page, section 2:
//               dL/dc_i = T_i a_i dL/dC, dL/da_i = T_i (c_i - C_{i+1}) dL/dC,
//               then through G to the conic and the 2D mean; the 2D mean
//               gradient has the sign of d G/d mu = G Sigma^-1 (x - mu)
//               (chain-rule page, mean-gradient formula).
//   preprocess  2D gradients to 3D mean, scale and quaternion by the chain
//   bwd         rule (CUDA-backward page, section 4): the conic gradient
//               through the matrix inverse, then (J W)^T G (J W) to Sigma3,
//               J's dependence on the camera-space mean (the perspective
//               nonlinearity), Sigma3 = L L^T with L = R diag(s), and the
//               quaternion normalisation.
//
// Two instantiations: Real = float is the "mirror" whose integer decisions
// (cull, radius, tile rectangle, depth key bits, contributor counts) are taken
// in fp32 like the kernels; Real = double is the gradient and
// finite-difference reference.  The float build must be compiled with
// -ffp-contract=off so that every operation below is one IEEE rounding.
//
// Readings of points the pages leave open are listed with the functions that
// use them.  Parity pins for every function live in tests/ (closed forms,
// invariants, brute force and float64 central differences with eps 1e-4).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// Camera and rasterizer parameters.  Field order is part of this oracle's own
// ctypes interface.
typedef struct oracle_camera {
    int width, height, tile;
    float fx, fy, cx, cy;
    float R[9];  // world -> camera rotation, row-major
    float t[3];  // world -> camera translation
    float z_near, eps2d, alpha_max, alpha_min, T_min, sigma_mult;
    float bg[3];
} oracle_camera;

}  // extern "C"

namespace {

template <typename Real>
struct Proj {
    Real u, v, depth;
    Real conic[3];
    int radius;
    int rect[4];  // x0, y0, x1, y1 (tile coordinates, half-open)
    unsigned touched;
};

// Unit quaternion (w, x, y, z) to rotation matrix, the textbook formula
// (training page, section D.4: R from a unit quaternion, det R = +1).
template <typename Real>
void quat_to_rot(Real w, Real x, Real y, Real z, Real R[3][3]) {
    Real xx = x * x, yy = y * y, zz = z * z;
    Real xy = x * y, xz = x * z, yz = y * z;
    Real wx = w * x, wy = w * y, wz = w * z;
    R[0][0] = Real(1) - Real(2) * (yy + zz);
    R[0][1] = Real(2) * (xy - wz);
    R[0][2] = Real(2) * (xz + wy);
    R[1][0] = Real(2) * (xy + wz);
    R[1][1] = Real(1) - Real(2) * (xx + zz);
    R[1][2] = Real(2) * (yz - wx);
    R[2][0] = Real(2) * (xz - wy);
    R[2][1] = Real(2) * (yz + wx);
    R[2][2] = Real(1) - Real(2) * (xx + yy);
}

// Per-Gaussian quantities the forward and the backward both need.
template <typename Real>
struct Geom {
    Real t[3];        // camera-space mean
    Real qn[4];       // normalised quaternion
    Real qnorm;       // |q|
    Real R[3][3];     // rotation of the Gaussian
    Real L[3][3];     // R diag(s)
    Real S3[3][3];    // Sigma3 = L L^T
    Real J[2][3];     // Jacobian of the pinhole projection at t
    Real M[2][3];     // J W
    Real S2[2][2];    // M Sigma3 M^T + eps I
};

template <typename Real>
bool geometry(const oracle_camera& cam, const Real* mu, const Real* s, const Real* q, Geom<Real>& g) {
    Real W[3][3];
    for (int i = 0; i < 3; ++i)
        for (int k = 0; k < 3; ++k) W[i][k] = Real(cam.R[3 * i + k]);
    for (int i = 0; i < 3; ++i)
        g.t[i] = ((W[i][0] * mu[0] + W[i][1] * mu[1]) + W[i][2] * mu[2]) + Real(cam.t[i]);
    // Near-plane cull (reading: z_near = 0.2, NaN depth also culled).
    if (!(g.t[2] > Real(cam.z_near))) return false;

    Real n2 = ((q[0] * q[0] + q[1] * q[1]) + q[2] * q[2]) + q[3] * q[3];
    if (!(n2 > Real(0))) return false;  // zero quaternion: no rotation defined
    g.qnorm = std::sqrt(n2);
    for (int k = 0; k < 4; ++k) g.qn[k] = q[k] / g.qnorm;
    quat_to_rot(g.qn[0], g.qn[1], g.qn[2], g.qn[3], g.R);

    for (int i = 0; i < 3; ++i)
        for (int k = 0; k < 3; ++k) g.L[i][k] = g.R[i][k] * s[k];
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j)
            g.S3[i][j] = (g.L[i][0] * g.L[j][0] + g.L[i][1] * g.L[j][1]) + g.L[i][2] * g.L[j][2];

    const Real tx = g.t[0], ty = g.t[1], tz = g.t[2];
    const Real fx = Real(cam.fx), fy = Real(cam.fy);
    const Real tz2 = tz * tz;
    g.J[0][0] = fx / tz;  g.J[0][1] = Real(0);  g.J[0][2] = -(fx * tx) / tz2;
    g.J[1][0] = Real(0);  g.J[1][1] = fy / tz;  g.J[1][2] = -(fy * ty) / tz2;
    for (int i = 0; i < 2; ++i)
        for (int k = 0; k < 3; ++k)
            g.M[i][k] = (g.J[i][0] * W[0][k] + g.J[i][1] * W[1][k]) + g.J[i][2] * W[2][k];
    Real T[2][3];
    for (int i = 0; i < 2; ++i)
        for (int k = 0; k < 3; ++k)
            T[i][k] = (g.M[i][0] * g.S3[0][k] + g.M[i][1] * g.S3[1][k]) + g.M[i][2] * g.S3[2][k];
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j)
            g.S2[i][j] = (T[i][0] * g.M[j][0] + T[i][1] * g.M[j][1]) + T[i][2] * g.M[j][2];
    // Low-pass dilation (reading: eps = 0.3 px^2 added to the diagonal).
    g.S2[0][0] = g.S2[0][0] + Real(cam.eps2d);
    g.S2[1][1] = g.S2[1][1] + Real(cam.eps2d);
    return true;
}

// Projection of one Gaussian.  Returns false (culled) when the Gaussian is
// behind the near plane, degenerate, non-finite or outside every tile.
template <typename Real>
bool project_one(const oracle_camera& cam, const Real* mu, const Real* s, const Real* q, Proj<Real>& p) {
    Geom<Real> g;
    if (!geometry(cam, mu, s, q, g)) return false;
    const Real a = g.S2[0][0], b = g.S2[0][1], c = g.S2[1][1];
    const Real det = a * c - b * b;
    if (!(det > Real(0))) return false;
    p.conic[0] = c / det;
    p.conic[1] = -b / det;
    p.conic[2] = a / det;
    // Largest eigenvalue of the 2x2 covariance; discriminant floored at 0.
    const Real mid = Real(0.5) * (a + c);
    const Real disc = mid * mid - det;
    const Real lam = mid + std::sqrt(std::max(disc, Real(0)));
    p.u = (Real(cam.fx) * g.t[0]) / g.t[2] + Real(cam.cx);
    p.v = (Real(cam.fy) * g.t[1]) / g.t[2] + Real(cam.cy);
    if (!std::isfinite(p.u) || !std::isfinite(p.v) || std::isnan(lam)) return false;
    // Support radius r = ceil(3 sqrt(lambda_max)) pixels, saturated at 2^24.
    Real rr = std::ceil(Real(cam.sigma_mult) * std::sqrt(lam));
    if (!(rr <= Real(16777216))) rr = Real(16777216);
    // Tile rectangle [x0, x1) x [y0, y1): floor/ceil of the AABB in tile units.
    const int TX = (cam.width + cam.tile - 1) / cam.tile;
    const int TY = (cam.height + cam.tile - 1) / cam.tile;
    const Real ts = Real(cam.tile);
    auto clampi = [](Real x, int hi) {
        if (x < Real(0)) x = Real(0);
        if (x > Real(hi)) x = Real(hi);
        return (int)x;
    };
    p.rect[0] = clampi(std::floor((p.u - rr) / ts), TX);
    p.rect[1] = clampi(std::floor((p.v - rr) / ts), TY);
    p.rect[2] = clampi(std::ceil((p.u + rr) / ts), TX);
    p.rect[3] = clampi(std::ceil((p.v + rr) / ts), TY);
    p.touched = (unsigned)((p.rect[2] - p.rect[0]) * (p.rect[3] - p.rect[1]));
    if (p.touched == 0) return false;
    p.radius = (int)rr;
    p.depth = g.t[2];
    return true;
}

template <typename Real>
void preprocess(const oracle_camera* cam, int N, const Real* means, const Real* scales, const Real* quats,
                const Real* opacity, Real* mean2d, Real* depth, Real* conic_opacity, int* radius, int* rect,
                unsigned* tiles_touched) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < N; ++i) {
        Proj<Real> p;
        bool vis = project_one(*cam, means + 3 * i, scales + 3 * i, quats + 4 * i, p);
        if (!vis) {
            mean2d[2 * i] = mean2d[2 * i + 1] = Real(0);
            depth[i] = Real(0);
            for (int k = 0; k < 4; ++k) conic_opacity[4 * i + k] = Real(0);
            radius[i] = 0;
            for (int k = 0; k < 4; ++k) rect[4 * i + k] = 0;
            tiles_touched[i] = 0;
            continue;
        }
        mean2d[2 * i] = p.u;
        mean2d[2 * i + 1] = p.v;
        depth[i] = p.depth;
        conic_opacity[4 * i + 0] = p.conic[0];
        conic_opacity[4 * i + 1] = p.conic[1];
        conic_opacity[4 * i + 2] = p.conic[2];
        conic_opacity[4 * i + 3] = opacity[i];
        radius[i] = p.radius;
        for (int k = 0; k < 4; ++k) rect[4 * i + k] = p.rect[k];
        tiles_touched[i] = p.touched;
    }
}

inline uint32_t float_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}

// Binning: every (tile, Gaussian) pair, sorted lexicographically by
// (tile, depth, id) (training page, section E.3: Gaussians are listed per
// tile and each tile's list is sorted by depth).  The pairs are grouped by
// tile (a count per tile, a prefix sum of the counts, then each Gaussian
// written into the groups of the tiles its rectangle covers), and every
// tile's group is sorted by (depth, id) with a plain comparison sort.  Tiles
// are independent, so their sorts run in parallel; the result is the same
// whatever the thread count.  ranges[t] = [first, last + 1) of tile t's
// group; an empty tile gets (0, 0).
template <typename Real>
long long bin(const oracle_camera* cam, int N, const Real* depth, const int* rect, const unsigned* tiles_touched,
              unsigned long long* keys, unsigned* ids, unsigned* ranges) {
    const int TX = (cam->width + cam->tile - 1) / cam->tile;
    const int TY = (cam->height + cam->tile - 1) / cam->tile;
    const int T = TX * TY;
    std::vector<size_t> count(T, 0), start(T + 1, 0);
    for (int i = 0; i < N; ++i) {
        if (tiles_touched[i] == 0) continue;
        const int* r = rect + 4 * i;
        for (int ty = r[1]; ty < r[3]; ++ty)
            for (int tx = r[0]; tx < r[2]; ++tx) ++count[ty * TX + tx];
    }
    for (int t = 0; t < T; ++t) start[t + 1] = start[t] + count[t];
    const size_t P = start[T];
    std::vector<std::pair<Real, uint32_t>> pairs(P);
    std::vector<size_t> cursor(start.begin(), start.end() - 1);
    for (int i = 0; i < N; ++i) {
        if (tiles_touched[i] == 0) continue;
        const int* r = rect + 4 * i;
        for (int ty = r[1]; ty < r[3]; ++ty)
            for (int tx = r[0]; tx < r[2]; ++tx) pairs[cursor[ty * TX + tx]++] = {depth[i], (uint32_t)i};
    }
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        std::sort(pairs.begin() + start[t], pairs.begin() + start[t + 1]);
        ranges[2 * t] = count[t] ? (unsigned)start[t] : 0u;
        ranges[2 * t + 1] = count[t] ? (unsigned)start[t + 1] : 0u;
        for (size_t k = start[t]; k < start[t + 1]; ++k) {
            if (ids) ids[k] = pairs[k].second;
            if (keys) {
                const float df = (float)pairs[k].first;
                keys[k] = ((unsigned long long)t << 32) | float_bits(df);
            }
        }
    }
    return (long long)P;
}

// Brute-force list of one tile: every Gaussian whose rectangle contains the
// tile, sorted by (depth, id).  Independent of the full binning above.
template <typename Real>
long long tile_list(const oracle_camera* cam, int N, const Real* depth, const int* rect, const unsigned* tiles_touched,
                    int tile, unsigned* out_ids) {
    const int TX = (cam->width + cam->tile - 1) / cam->tile;
    const int tx = tile % TX, ty = tile / TX;
    std::vector<std::pair<Real, uint32_t>> v;
    for (int i = 0; i < N; ++i) {
        if (tiles_touched[i] == 0) continue;
        const int* r = rect + 4 * i;
        if (tx >= r[0] && tx < r[2] && ty >= r[1] && ty < r[3]) v.emplace_back(depth[i], (uint32_t)i);
    }
    std::sort(v.begin(), v.end());
    if (out_ids)
        for (size_t k = 0; k < v.size(); ++k) out_ids[k] = v[k].second;
    return (long long)v.size();
}

// exp for the fp32 mirror: the float result must be the one the kernels
// compute, because a one-ulp difference in exp can flip an alpha_min or T_min
// decision.  A fixed sequence of IEEE operations that any machine with a
// correctly rounded fma reproduces: clamp x to >= -87; n = rint(x log2 e)
// through the 1.5 * 2^23 shifter; f = x log2 e - n with log2 e split into a
// high and a low part (two fused multiply-adds);
// 2^f = sum_{k<=7} (ln 2)^k f^k / k! (Taylor series of exp(f ln 2), Horner
// with fused multiply-adds); scale by 2^n through the exponent bits.
// Argument reduction after Cody and Waite.  Pinned against float64 exp.
inline float exp_mirror(float x) {
    x = std::fmax(x, -87.0f);
    const float t = std::fma(x, 0x1.715476p+0f, 0x1.8p+23f);
    const float n = t - 0x1.8p+23f;
    float f = std::fma(x, 0x1.715476p+0f, -n);
    f = std::fma(x, 0x1.4ae0c0p-26f, f);
    float p = 0x1.ffcbfcp-17f;
    p = std::fma(p, f, 0x1.430912p-13f);
    p = std::fma(p, f, 0x1.5d87fep-10f);
    p = std::fma(p, f, 0x1.3b2ab6p-7f);
    p = std::fma(p, f, 0x1.c6b08ep-5f);
    p = std::fma(p, f, 0x1.ebfbe0p-3f);
    p = std::fma(p, f, 0x1.62e430p-1f);
    p = std::fma(p, f, 1.0f);
    uint32_t tb, sb, pb;
    const float shift = 0x1.8p+23f;
    std::memcpy(&tb, &t, 4);
    std::memcpy(&sb, &shift, 4);
    std::memcpy(&pb, &p, 4);
    pb += (tb - sb) << 23;
    float r;
    std::memcpy(&r, &pb, 4);
    return r;
}
inline float oexp(float x) { return exp_mirror(x); }
inline double oexp(double x) { return std::exp(x); }

// Evaluation of one (pixel, Gaussian) term of the compositing sum.
template <typename Real>
struct Term {
    Real dx, dy, G, at, alpha;
    bool used;  // passes the power > 0 and alpha < alpha_min skips
};

template <typename Real>
inline Term<Real> eval_term(const oracle_camera& cam, Real px, Real py, const Real* xy, const Real* co) {
    Term<Real> e;
    e.dx = px - xy[0];
    e.dy = py - xy[1];
    // power = -1/2 d^T A d, with d^T A d = a dx^2 + 2 b dx dy + c dy^2 taken as
    // fma(2 b dx, dy, fma(a dx, dx, c dy dy)): in fp32 this fixes every
    // rounding, so the alpha_min / T_min decisions match the kernels'.
    const Real qc = (co[2] * e.dy) * e.dy;
    const Real q = std::fma(Real(2) * co[1] * e.dx, e.dy, std::fma(co[0] * e.dx, e.dx, qc));
    const Real power = Real(-0.5) * q;
    e.used = false;
    e.G = e.at = e.alpha = Real(0);
    if (power > Real(0)) return e;  // only for a non positive-definite conic
    e.G = oexp(power);
    e.at = co[3] * e.G;
    e.alpha = std::min(Real(cam.alpha_max), e.at);
    if (e.alpha < Real(cam.alpha_min)) return e;  // reading: alpha_min = 1/255
    e.used = true;
    return e;
}

template <typename Real>
void tiles_of(const oracle_camera* cam, const int* subset, int n_subset, std::vector<int>& out) {
    const int TX = (cam->width + cam->tile - 1) / cam->tile;
    const int TY = (cam->height + cam->tile - 1) / cam->tile;
    out.clear();
    if (subset) {
        out.assign(subset, subset + n_subset);
    } else {
        for (int t = 0; t < TX * TY; ++t) out.push_back(t);
    }
}

// Forward compositing, front to back.  Reading: the Gaussian whose blend would
// take T below T_min stops the pixel and is not blended; n_contrib is the
// list position (within the tile) of the last blended Gaussian plus one.
template <typename Real>
void render_fwd(const oracle_camera* cam, const unsigned* ranges, const unsigned* ids, const Real* mean2d,
                const Real* conic_opacity, const Real* colors, Real* image, Real* final_T, unsigned* n_contrib,
                unsigned* n_eval, unsigned* n_blend, unsigned* blend_mask, const int* subset, int n_subset) {
    const int W = cam->width, H = cam->height, TS = cam->tile;
    const int TX = (W + TS - 1) / TS;
    std::vector<int> tiles;
    tiles_of<Real>(cam, subset, n_subset, tiles);
#pragma omp parallel for schedule(dynamic, 4)
    for (long long it = 0; it < (long long)tiles.size(); ++it) {
        const int tile = tiles[it];
        const int tx = tile % TX, ty = tile / TX;
        const unsigned r0 = ranges[2 * tile], r1 = ranges[2 * tile + 1];
        for (int y = ty * TS; y < std::min(H, ty * TS + TS); ++y) {
            for (int x = tx * TS; x < std::min(W, tx * TS + TS); ++x) {
                const Real px = Real(x) + Real(0.5), py = Real(y) + Real(0.5);
                Real T = Real(1), C[3] = {Real(0), Real(0), Real(0)};
                unsigned last = 0, evals = 0, blended = 0;
                for (unsigned k = r0; k < r1; ++k) {
                    const unsigned j = ids[k];
                    ++evals;
                    Term<Real> e = eval_term(*cam, px, py, mean2d + 2 * j, conic_opacity + 4 * j);
                    if (!e.used) continue;
                    const Real Tn = T * (Real(1) - e.alpha);
                    if (Tn < Real(cam->T_min)) break;
                    for (int ch = 0; ch < 3; ++ch) C[ch] += colors[3 * j + ch] * e.alpha * T;
                    T = Tn;
                    last = k - r0 + 1;
                    ++blended;
                    if (blend_mask) {
                        // bit k of the 8x8 quadrant of the tile this pixel lies in
                        const unsigned quad = (unsigned)(((y % TS) / 8) * 2 + ((x % TS) / 8));
                        unsigned* word = blend_mask + (size_t)(k >> 5) * 4 + quad;
                        const unsigned bit = 1u << (k & 31u);
#pragma omp atomic
                        *word |= bit;
                    }
                }
                const size_t pix = (size_t)y * W + x;
                for (int ch = 0; ch < 3; ++ch) image[(size_t)ch * H * W + pix] = C[ch] + T * Real(cam->bg[ch]);
                final_T[pix] = T;
                n_contrib[pix] = last;
                if (n_eval) n_eval[pix] = evals;
                if (n_blend) n_blend[pix] = blended;
            }
        }
    }
}

// Backward of the compositing for one tile.  For each pixel the forward is
// re-run to list the blended terms with their transmittance T_k (computed as
// the product of (1 - alpha) over the terms in front, as defined), then the
// colour behind each term is built back to front: S = bg at the back and
// S <- alpha_k c_k + (1 - alpha_k) S.  dL/dalpha_k = T_k (c_k - S_k) . g.
// Reading: the derivative through the 0.99 cap is the exact one (zero when
// the cap is active).  Gradients w.r.t. the conic are w.r.t. its three
// unique entries (a, b, c) of a dx^2 + 2 b dx dy + c dy^2.
template <typename Real>
void render_bwd_tile(const oracle_camera* cam, int tile, const unsigned* ranges, const unsigned* ids,
                     const Real* mean2d, const Real* conic_opacity, const Real* colors, const Real* dL_dimage,
                     std::vector<Real>& local /* 9 per list entry */) {
    const int W = cam->width, H = cam->height, TS = cam->tile;
    const int TX = (W + TS - 1) / TS;
    const int tx = tile % TX, ty = tile / TX;
    const unsigned r0 = ranges[2 * tile], r1 = ranges[2 * tile + 1];
    local.assign((size_t)(r1 - r0) * 9, Real(0));
    struct Blended { unsigned k; Term<Real> e; Real T; };
    std::vector<Blended> bl;
    for (int y = ty * TS; y < std::min(H, ty * TS + TS); ++y) {
        for (int x = tx * TS; x < std::min(W, tx * TS + TS); ++x) {
            const Real px = Real(x) + Real(0.5), py = Real(y) + Real(0.5);
            bl.clear();
            Real T = Real(1);
            for (unsigned k = r0; k < r1; ++k) {
                const unsigned j = ids[k];
                Term<Real> e = eval_term(*cam, px, py, mean2d + 2 * j, conic_opacity + 4 * j);
                if (!e.used) continue;
                const Real Tn = T * (Real(1) - e.alpha);
                if (Tn < Real(cam->T_min)) break;
                bl.push_back({k, e, T});
                T = Tn;
            }
            const size_t pix = (size_t)y * W + x;
            Real g[3], S[3];
            for (int ch = 0; ch < 3; ++ch) {
                g[ch] = dL_dimage[(size_t)ch * H * W + pix];
                S[ch] = Real(cam->bg[ch]);
            }
            for (size_t m = bl.size(); m-- > 0;) {
                const Blended& b = bl[m];
                const unsigned j = ids[b.k];
                const Real* co = conic_opacity + 4 * j;
                const Real* c = colors + 3 * j;
                Real* acc = local.data() + (size_t)(b.k - r0) * 9;
                Real dL_dalpha = Real(0);
                for (int ch = 0; ch < 3; ++ch) {
                    acc[6 + ch] += b.e.alpha * b.T * g[ch];          // dL/dc
                    dL_dalpha += (c[ch] - S[ch]) * g[ch];
                }
                dL_dalpha *= b.T;
                for (int ch = 0; ch < 3; ++ch) S[ch] = b.e.alpha * c[ch] + (Real(1) - b.e.alpha) * S[ch];
                Real dL_dsigma = Real(0), dL_dG = Real(0);
                if (b.e.at <= Real(cam->alpha_max)) {
                    dL_dsigma = b.e.G * dL_dalpha;
                    dL_dG = co[3] * dL_dalpha;
                }
                const Real h = b.e.G * dL_dG;  // dL/dpower
                const Real dx = b.e.dx, dy = b.e.dy;
                acc[0] += (co[0] * dx + co[1] * dy) * h;              // dL/du
                acc[1] += (co[1] * dx + co[2] * dy) * h;              // dL/dv
                acc[2] += Real(-0.5) * dx * dx * h;                    // dL/da
                acc[3] += -dx * dy * h;                                 // dL/db
                acc[4] += Real(-0.5) * dy * dy * h;                    // dL/dc
                acc[5] += dL_dsigma;                                    // dL/dsigma
            }
        }
    }
}

template <typename Real>
void render_bwd(const oracle_camera* cam, int N, const unsigned* ranges, const unsigned* ids, const Real* mean2d,
                const Real* conic_opacity, const Real* colors, const Real* dL_dimage, Real* dL_dmean2d,
                Real* dL_dconic_opacity, Real* dL_dcolor, const int* subset, int n_subset) {
    for (size_t i = 0; i < (size_t)N * 2; ++i) dL_dmean2d[i] = Real(0);
    for (size_t i = 0; i < (size_t)N * 4; ++i) dL_dconic_opacity[i] = Real(0);
    for (size_t i = 0; i < (size_t)N * 3; ++i) dL_dcolor[i] = Real(0);
    std::vector<int> tiles;
    tiles_of<Real>(cam, subset, n_subset, tiles);
    // Tiles are processed in groups; each group's per-tile partial sums are
    // added to the outputs in tile order, so the result does not depend on
    // the number of threads.
    const int GROUP = 256;
    std::vector<std::vector<Real>> locals(GROUP);
    for (size_t g0 = 0; g0 < tiles.size(); g0 += GROUP) {
        const int ng = (int)std::min((size_t)GROUP, tiles.size() - g0);
#pragma omp parallel for schedule(dynamic, 1)
        for (int gi = 0; gi < ng; ++gi)
            render_bwd_tile(cam, tiles[g0 + gi], ranges, ids, mean2d, conic_opacity, colors, dL_dimage, locals[gi]);
        for (int gi = 0; gi < ng; ++gi) {
            const int tile = tiles[g0 + gi];
            const unsigned r0 = ranges[2 * tile], r1 = ranges[2 * tile + 1];
            for (unsigned k = r0; k < r1; ++k) {
                const unsigned j = ids[k];
                const Real* a = locals[gi].data() + (size_t)(k - r0) * 9;
                dL_dmean2d[2 * j] += a[0];
                dL_dmean2d[2 * j + 1] += a[1];
                dL_dconic_opacity[4 * j + 0] += a[2];
                dL_dconic_opacity[4 * j + 1] += a[3];
                dL_dconic_opacity[4 * j + 2] += a[4];
                dL_dconic_opacity[4 * j + 3] += a[5];
                dL_dcolor[3 * j + 0] += a[6];
                dL_dcolor[3 * j + 1] += a[7];
                dL_dcolor[3 * j + 2] += a[8];
            }
        }
    }
}

// d R / d (w, x, y, z) contracted with G_R: the derivative of the textbook
// quaternion matrix, entry by entry.
template <typename Real>
void rot_backward(const Real q[4], const Real GR[3][3], Real dq[4]) {
    const Real w = q[0], x = q[1], y = q[2], z = q[3];
    // R00 = 1 - 2(y^2 + z^2)
    Real dw = 0, dx = 0, dy = 0, dz = 0;
    dy += -4 * y * GR[0][0];  dz += -4 * z * GR[0][0];
    // R01 = 2(xy - wz)
    dx += 2 * y * GR[0][1];  dy += 2 * x * GR[0][1];  dw += -2 * z * GR[0][1];  dz += -2 * w * GR[0][1];
    // R02 = 2(xz + wy)
    dx += 2 * z * GR[0][2];  dz += 2 * x * GR[0][2];  dw += 2 * y * GR[0][2];  dy += 2 * w * GR[0][2];
    // R10 = 2(xy + wz)
    dx += 2 * y * GR[1][0];  dy += 2 * x * GR[1][0];  dw += 2 * z * GR[1][0];  dz += 2 * w * GR[1][0];
    // R11 = 1 - 2(x^2 + z^2)
    dx += -4 * x * GR[1][1];  dz += -4 * z * GR[1][1];
    // R12 = 2(yz - wx)
    dy += 2 * z * GR[1][2];  dz += 2 * y * GR[1][2];  dw += -2 * x * GR[1][2];  dx += -2 * w * GR[1][2];
    // R20 = 2(xz - wy)
    dx += 2 * z * GR[2][0];  dz += 2 * x * GR[2][0];  dw += -2 * y * GR[2][0];  dy += -2 * w * GR[2][0];
    // R21 = 2(yz + wx)
    dy += 2 * z * GR[2][1];  dz += 2 * y * GR[2][1];  dw += 2 * x * GR[2][1];  dx += 2 * w * GR[2][1];
    // R22 = 1 - 2(x^2 + y^2)
    dx += -4 * x * GR[2][2];  dy += -4 * y * GR[2][2];
    dq[0] = dw; dq[1] = dx; dq[2] = dy; dq[3] = dz;
}

// Chain rule from the 2D quantities (mean2d, conic, opacity, colour) to the
// 3D parameters.  Accumulates (+=) so that several cameras can sum.
template <typename Real>
void preprocess_bwd(const oracle_camera* cam, int N, const Real* means, const Real* scales, const Real* quats,
                    const int* radius, const Real* dL_dmean2d, const Real* dL_dconic_opacity,
                    const Real* dL_dcolor2d, Real* dL_dmeans, Real* dL_dscales, Real* dL_dquats,
                    Real* dL_dopacity, Real* dL_dcolors, Real* grad2d_accum, unsigned* vis_count) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < N; ++i) {
        if (radius[i] == 0) continue;  // culled: exactly zero gradient
        // Densification statistics (training page, section D.1: the position
        // gradient accumulated over views): |dL/dmean2d| of this view, and the
        // number of views in which the Gaussian is visible.
        if (grad2d_accum) {
            const Real gx = dL_dmean2d[2 * i], gy = dL_dmean2d[2 * i + 1];
            grad2d_accum[i] += std::sqrt(gx * gx + gy * gy);
            vis_count[i] += 1;
        }
        Geom<Real> g;
        if (!geometry(*cam, means + 3 * i, scales + 3 * i, quats + 4 * i, g)) continue;
        const Real* s = scales + 3 * i;
        // Conic A = Sigma2^-1.
        const Real a = g.S2[0][0], b = g.S2[0][1], c = g.S2[1][1];
        const Real det = a * c - b * b;
        const Real A[2][2] = {{c / det, -b / det}, {-b / det, a / det}};
        // dL/dA as a symmetric matrix: the off-diagonal unique entry appears twice.
        const Real* gA = dL_dconic_opacity + 4 * i;
        const Real GA[2][2] = {{gA[0], Real(0.5) * gA[1]}, {Real(0.5) * gA[1], gA[2]}};
        // dL/dSigma2 = -A^T GA A^T (derivative of the matrix inverse).
        Real tmp[2][2], G2[2][2];
        for (int r = 0; r < 2; ++r)
            for (int k = 0; k < 2; ++k) tmp[r][k] = A[r][0] * GA[0][k] + A[r][1] * GA[1][k];
        for (int r = 0; r < 2; ++r)
            for (int k = 0; k < 2; ++k) G2[r][k] = -(tmp[r][0] * A[0][k] + tmp[r][1] * A[1][k]);
        // dL/dSigma3 = M^T G2 M.
        Real G3[3][3];
        for (int r = 0; r < 3; ++r)
            for (int k = 0; k < 3; ++k) {
                Real acc = 0;
                for (int p = 0; p < 2; ++p)
                    for (int q2 = 0; q2 < 2; ++q2) acc += g.M[p][r] * G2[p][q2] * g.M[q2][k];
                G3[r][k] = acc;
            }
        // dL/dM = 2 G2 M Sigma3 ; dL/dJ = dL/dM W^T.
        Real GM[2][3], GJ[2][3];
        for (int r = 0; r < 2; ++r)
            for (int k = 0; k < 3; ++k) {
                Real acc = 0;
                for (int p = 0; p < 2; ++p)
                    for (int m = 0; m < 3; ++m) acc += G2[r][p] * g.M[p][m] * g.S3[m][k];
                GM[r][k] = Real(2) * acc;
            }
        for (int r = 0; r < 2; ++r)
            for (int k = 0; k < 3; ++k) {
                Real acc = 0;
                for (int m = 0; m < 3; ++m) acc += GM[r][m] * Real(cam->R[3 * k + m]);
                GJ[r][k] = acc;
            }
        // Camera-space mean: through the projected mean and through J.
        const Real tx = g.t[0], ty = g.t[1], tz = g.t[2];
        const Real fx = Real(cam->fx), fy = Real(cam->fy);
        const Real gu = dL_dmean2d[2 * i], gv = dL_dmean2d[2 * i + 1];
        Real dt[3] = {0, 0, 0};
        dt[0] += fx / tz * gu;
        dt[1] += fy / tz * gv;
        dt[2] += -fx * tx / (tz * tz) * gu - fy * ty / (tz * tz) * gv;
        dt[2] += -fx / (tz * tz) * GJ[0][0];
        dt[0] += -fx / (tz * tz) * GJ[0][2];
        dt[2] += Real(2) * fx * tx / (tz * tz * tz) * GJ[0][2];
        dt[2] += -fy / (tz * tz) * GJ[1][1];
        dt[1] += -fy / (tz * tz) * GJ[1][2];
        dt[2] += Real(2) * fy * ty / (tz * tz * tz) * GJ[1][2];
        for (int k = 0; k < 3; ++k) {
            Real acc = 0;
            for (int r = 0; r < 3; ++r) acc += Real(cam->R[3 * r + k]) * dt[r];
            dL_dmeans[3 * i + k] += acc;
        }
        // Sigma3 = L L^T, L = R diag(s).
        Real GL[3][3], GR[3][3];
        for (int r = 0; r < 3; ++r)
            for (int k = 0; k < 3; ++k) {
                Real acc = 0;
                for (int m = 0; m < 3; ++m) acc += G3[r][m] * g.L[m][k];
                GL[r][k] = Real(2) * acc;
            }
        for (int k = 0; k < 3; ++k) {
            Real acc = 0;
            for (int r = 0; r < 3; ++r) acc += GL[r][k] * g.R[r][k];
            dL_dscales[3 * i + k] += acc;
        }
        for (int r = 0; r < 3; ++r)
            for (int k = 0; k < 3; ++k) GR[r][k] = GL[r][k] * s[k];
        Real dqn[4];
        rot_backward(g.qn, GR, dqn);
        // Through q_hat = q / |q|.
        const Real proj = ((g.qn[0] * dqn[0] + g.qn[1] * dqn[1]) + g.qn[2] * dqn[2]) + g.qn[3] * dqn[3];
        for (int k = 0; k < 4; ++k) dL_dquats[4 * i + k] += (dqn[k] - g.qn[k] * proj) / g.qnorm;
        dL_dopacity[i] += gA[3];
        for (int ch = 0; ch < 3; ++ch) dL_dcolors[3 * i + ch] += dL_dcolor2d[3 * i + ch];
    }
}

// ---------------------------------------------------------------------------
// Colour from real spherical harmonics ("Gaussian Splatting反向传播的CUDA实现",
// section 4: the colour gradient reaches the SH coefficients through the
// derivative of the SH basis, band-limited).  Reading: the orthonormal real SH
// of degree <= 3 in Cartesian form on the unit view direction d = (x, y, z),
// coefficients ordered k = l^2 + l + m; colour = max(0, sum_k Y_k(d) sh_k +
// offset) per channel, d = normalise(mean - camera centre), camera centre
// = -R^T t.  The clamp at 0 is the constraint; its derivative is 0 where it
// is active.
// ---------------------------------------------------------------------------
template <typename Real>
void sh_basis(const Real d[3], int degree, Real Y[16], Real dY[16][3]) {
    const Real x = d[0], y = d[1], z = d[2];
    const Real C0 = Real(0.28209479177387814), C1 = Real(0.4886025119029199);
    const Real C2a = Real(1.0925484305920792), C2b = Real(0.31539156525252005), C2c = Real(0.5462742152960396);
    const Real C3a = Real(0.5900435899266435), C3b = Real(2.890611442640554), C3c = Real(0.4570457994644658);
    const Real C3d = Real(0.3731763325901154), C3e = Real(1.445305721320277);
    for (int k = 0; k < 16; ++k) {
        Y[k] = Real(0);
        dY[k][0] = dY[k][1] = dY[k][2] = Real(0);
    }
    Y[0] = C0;
    if (degree < 1) return;
    Y[1] = C1 * y;  dY[1][1] = C1;
    Y[2] = C1 * z;  dY[2][2] = C1;
    Y[3] = C1 * x;  dY[3][0] = C1;
    if (degree < 2) return;
    Y[4] = C2a * x * y;               dY[4][0] = C2a * y;  dY[4][1] = C2a * x;
    Y[5] = C2a * y * z;               dY[5][1] = C2a * z;  dY[5][2] = C2a * y;
    Y[6] = C2b * (3 * z * z - 1);     dY[6][2] = C2b * 6 * z;
    Y[7] = C2a * x * z;               dY[7][0] = C2a * z;  dY[7][2] = C2a * x;
    Y[8] = C2c * (x * x - y * y);     dY[8][0] = C2c * 2 * x;  dY[8][1] = -C2c * 2 * y;
    if (degree < 3) return;
    Y[9] = C3a * y * (3 * x * x - y * y);
    dY[9][0] = C3a * 6 * x * y;  dY[9][1] = C3a * (3 * x * x - 3 * y * y);
    Y[10] = C3b * x * y * z;
    dY[10][0] = C3b * y * z;  dY[10][1] = C3b * x * z;  dY[10][2] = C3b * x * y;
    Y[11] = C3c * y * (5 * z * z - 1);
    dY[11][1] = C3c * (5 * z * z - 1);  dY[11][2] = C3c * 10 * y * z;
    Y[12] = C3d * z * (5 * z * z - 3);
    dY[12][2] = C3d * (15 * z * z - 3);
    Y[13] = C3c * x * (5 * z * z - 1);
    dY[13][0] = C3c * (5 * z * z - 1);  dY[13][2] = C3c * 10 * x * z;
    Y[14] = C3e * z * (x * x - y * y);
    dY[14][0] = C3e * 2 * x * z;  dY[14][1] = -C3e * 2 * y * z;  dY[14][2] = C3e * (x * x - y * y);
    Y[15] = C3a * x * (x * x - 3 * y * y);
    dY[15][0] = C3a * (3 * x * x - 3 * y * y);  dY[15][1] = -C3a * 6 * x * y;
}

template <typename Real>
void view_dir(const oracle_camera& cam, const Real* mu, Real v[3], Real d[3], Real& norm) {
    for (int j = 0; j < 3; ++j) {
        Real c = 0;
        for (int i = 0; i < 3; ++i) c -= Real(cam.R[3 * i + j]) * Real(cam.t[i]);  // camera centre -R^T t
        v[j] = mu[j] - c;
    }
    norm = std::sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2]);
    for (int j = 0; j < 3; ++j) d[j] = v[j] / norm;
}

template <typename Real>
void sh_fwd(const oracle_camera* cam, int N, int degree, int K, const Real* means, const Real* sh, Real offset,
            Real* colors) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < N; ++i) {
        Real v[3], d[3], nrm, Y[16], dY[16][3];
        view_dir(*cam, means + 3 * i, v, d, nrm);
        sh_basis(d, degree, Y, dY);
        const int nk = (degree + 1) * (degree + 1);
        for (int ch = 0; ch < 3; ++ch) {
            Real acc = 0;
            for (int k = 0; k < nk; ++k) acc += Y[k] * sh[((size_t)i * K + k) * 3 + ch];
            colors[3 * i + ch] = std::max(acc + offset, Real(0));
        }
    }
}

template <typename Real>
void sh_bwd(const oracle_camera* cam, int N, int degree, int K, const Real* means, const Real* sh, Real offset,
            const Real* dL_dcolors, Real* dL_dsh, Real* dL_dmeans) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < N; ++i) {
        Real v[3], d[3], nrm, Y[16], dY[16][3];
        view_dir(*cam, means + 3 * i, v, d, nrm);
        sh_basis(d, degree, Y, dY);
        const int nk = (degree + 1) * (degree + 1);
        Real g[3];
        for (int ch = 0; ch < 3; ++ch) {
            Real acc = 0;
            for (int k = 0; k < nk; ++k) acc += Y[k] * sh[((size_t)i * K + k) * 3 + ch];
            g[ch] = (acc + offset > Real(0)) ? dL_dcolors[3 * i + ch] : Real(0);  // clamp active: no gradient
        }
        Real dd[3] = {0, 0, 0};  // dL/d(direction), treating (x, y, z) as free
        for (int k = 0; k < nk; ++k) {
            Real s = 0;
            for (int ch = 0; ch < 3; ++ch) {
                dL_dsh[((size_t)i * K + k) * 3 + ch] += Y[k] * g[ch];
                s += sh[((size_t)i * K + k) * 3 + ch] * g[ch];
            }
            for (int j = 0; j < 3; ++j) dd[j] += dY[k][j] * s;
        }
        // d = v / |v|: dL/dv = (I - d d^T) dL/dd / |v|, and v = mean - centre
        const Real dot = d[0] * dd[0] + d[1] * dd[1] + d[2] * dd[2];
        for (int j = 0; j < 3; ++j) dL_dmeans[3 * i + j] += (dd[j] - d[j] * dot) / nrm;
    }
}

template <typename Real>
void sh_basis_eval(int n, const Real* dirs, Real* out) {
    for (int i = 0; i < n; ++i) {
        Real Y[16], dY[16][3];
        sh_basis(dirs + 3 * i, 3, Y, dY);
        for (int k = 0; k < 16; ++k) out[16 * i + k] = Y[k];
    }
}

}  // namespace

extern "C" {

void oracle_exp_f32(const float* x, float* y, long long n) {
    for (long long i = 0; i < n; ++i) y[i] = exp_mirror(x[i]);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

#define ORACLE_BOTH(MACRO) MACRO(float, f32) MACRO(double, f64)

#define DEF_PRE(R, SUF)                                                                                       \
    void oracle_preprocess_##SUF(const oracle_camera* cam, int N, const R* means, const R* scales,           \
                                 const R* quats, const R* opacity, R* mean2d, R* depth, R* conic_opacity,    \
                                 int* radius, int* rect, unsigned* tiles_touched) {                          \
        preprocess<R>(cam, N, means, scales, quats, opacity, mean2d, depth, conic_opacity, radius, rect,     \
                      tiles_touched);                                                                        \
    }                                                                                                        \
    long long oracle_bin_##SUF(const oracle_camera* cam, int N, const R* depth, const int* rect,             \
                               const unsigned* tiles_touched, unsigned long long* keys, unsigned* ids,       \
                               unsigned* ranges) {                                                           \
        return bin<R>(cam, N, depth, rect, tiles_touched, keys, ids, ranges);                                \
    }                                                                                                        \
    long long oracle_tile_list_##SUF(const oracle_camera* cam, int N, const R* depth, const int* rect,       \
                                     const unsigned* tiles_touched, int tile, unsigned* out_ids) {           \
        return tile_list<R>(cam, N, depth, rect, tiles_touched, tile, out_ids);                              \
    }                                                                                                        \
    void oracle_render_fwd_##SUF(const oracle_camera* cam, const unsigned* ranges, const unsigned* ids,      \
                                 const R* mean2d, const R* conic_opacity, const R* colors, R* image,         \
                                 R* final_T, unsigned* n_contrib, unsigned* n_eval, unsigned* n_blend,       \
                                 unsigned* blend_mask, const int* subset, int n_subset) {                    \
        render_fwd<R>(cam, ranges, ids, mean2d, conic_opacity, colors, image, final_T, n_contrib, n_eval,    \
                      n_blend, blend_mask, subset, n_subset);                                                \
    }                                                                                                        \
    void oracle_render_bwd_##SUF(const oracle_camera* cam, int N, const unsigned* ranges, const unsigned* ids, \
                                 const R* mean2d, const R* conic_opacity, const R* colors,                   \
                                 const R* dL_dimage, R* dL_dmean2d, R* dL_dconic_opacity, R* dL_dcolor,      \
                                 const int* subset, int n_subset) {                                          \
        render_bwd<R>(cam, N, ranges, ids, mean2d, conic_opacity, colors, dL_dimage, dL_dmean2d,             \
                      dL_dconic_opacity, dL_dcolor, subset, n_subset);                                       \
    }                                                                                                        \
    void oracle_preprocess_bwd_##SUF(const oracle_camera* cam, int N, const R* means, const R* scales,       \
                                     const R* quats, const int* radius, const R* dL_dmean2d,                 \
                                     const R* dL_dconic_opacity, const R* dL_dcolor2d, R* dL_dmeans,         \
                                     R* dL_dscales, R* dL_dquats, R* dL_dopacity, R* dL_dcolors,             \
                                     R* grad2d_accum, unsigned* vis_count) {                                 \
        preprocess_bwd<R>(cam, N, means, scales, quats, radius, dL_dmean2d, dL_dconic_opacity, dL_dcolor2d,  \
                          dL_dmeans, dL_dscales, dL_dquats, dL_dopacity, dL_dcolors, grad2d_accum,           \
                          vis_count);                                                                        \
    }

ORACLE_BOTH(DEF_PRE)

#define DEF_SH(R, SUF)                                                                                        \
    void oracle_sh_fwd_##SUF(const oracle_camera* cam, int N, int degree, int K, const R* means, const R* sh, \
                             R offset, R* colors) {                                                          \
        sh_fwd<R>(cam, N, degree, K, means, sh, offset, colors);                                             \
    }                                                                                                        \
    void oracle_sh_bwd_##SUF(const oracle_camera* cam, int N, int degree, int K, const R* means, const R* sh, \
                             R offset, const R* dL_dcolors, R* dL_dsh, R* dL_dmeans) {                       \
        sh_bwd<R>(cam, N, degree, K, means, sh, offset, dL_dcolors, dL_dsh, dL_dmeans);                      \
    }                                                                                                        \
    void oracle_sh_basis_##SUF(int n, const R* dirs, R* out) { sh_basis_eval<R>(n, dirs, out); }

ORACLE_BOTH(DEF_SH)

}  // extern "C"
