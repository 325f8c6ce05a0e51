// Tile binning and (tile, depth) ordering.
//
// "4-3DGS训练与优化" section E.3: each projected Gaussian's AABB selects the
// tiles it may touch; the Gaussians of each tile are sorted by depth and
// splatted in that order; tiles are independent.  "Gaussian Splatting反向传播的
// CUDA实现" section 1: the sorted list and the per-tile ranges are kept and
// reused by the backward.
//
// The order produced is that of a sort of 64-bit keys (tile << 32 |
// float_bits(depth)) with ties broken by Gaussian id, reached without ever
// sorting the (tile, Gaussian) pairs:
//   1. the N Gaussians are sorted by depth bits (stable LSD radix sort, 8-bit
//      digits, ids in increasing order initially, culled ones last), which
//      gives every visible Gaussian its (depth, id) rank;
//   2. cell route (images of at most 1024 x 1024 tiles): the (cell,
//      Gaussian) pairs of 4 x 4-tile cells are stably sorted by cell, and
//      each cell's rank-ordered list is expanded into its 16 tiles' lists
//      (see "Super-tile binning" below);
//   3. wide-image route (otherwise): the (tile, Gaussian) pairs are emitted
//      in rank order and stably sorted by tile id alone (ceil(log2 T) bits,
//      at most 8 per pass), ranges found by comparing neighbours.
// A stable sort by tile (or cell) of a list already in (depth, id) order
// keeps that order within each tile, so both routes give the 64-bit sort's
// result.
//
// Every kernel is a plain grid over its data; there are no inter-block waits.

#include <cuda_runtime.h>

#include "gs_internal.cuh"
#include "pdl.cuh"

namespace gs {
namespace {

constexpr int kSortBlock = 256;
constexpr int kSortMaxGrid = 148 * 4;  // CTAs per radix pass: a multiple of the SM count
constexpr int kRadixMax = 256;
constexpr int kScanGroup = 32;         // chunks per group of the per-group digit totals
constexpr int kMaxGroups = (kSortMaxGrid + kScanGroup - 1) / kScanGroup;
constexpr int kMaxPasses = 8;          // 4 depth passes + up to 3 tile passes (+1 spare)
constexpr int kScanItems = 8;          // items per thread in the rank-order scan
constexpr int kScanTile = kSortBlock * kScanItems;
constexpr int kFusedMaxBits = 8;       // fused binning: TX and TY at most 256

struct SortMisc {
    unsigned n_gauss;    // N
    unsigned p_eff;      // P if it fits the capacity, else 0
    unsigned ps;         // super-tile pairs if P fits the capacity, else 0
    unsigned nseg;       // segments of the super-tile lists
    unsigned pad[60];
};

struct BinWs {
    WsHeader* hdr;
    SortMisc* misc;
    unsigned *dkeys0, *dvals0, *dkeys1, *dvals1;  // depth sort, N each
    unsigned* pair_off;                            // N + 1
    unsigned* cnt_rank;                            // N: pairs of each rank (written by the scan's first kernel)
    unsigned* scan_part;                           // ceil(N / kScanTile) + 1
    unsigned *tkeys0, *tvals0, *tkeys1, *tvals1;   // pair sort, capacity each
    unsigned* hist;                                // kMaxPasses * kSortMaxGrid * kRadixMax (chunk-major)
    unsigned* totals;                              // kMaxPasses * kRadixMax
    unsigned* gtot;                                // kMaxPasses * kMaxGroups * kRadixMax (group-major)
    // super-tile route only (empty otherwise)
    unsigned* rc_rank;                             // N packed super-tile rectangles in rank order
    unsigned char* sub_rank;                       // N: the tile rectangle's offsets in its edge cells (sub_offsets)
    unsigned *owner_lo, *owner_hi;                 // kSortMaxGrid each: ranks owning chunk ends
    unsigned* cell_ranges;                         // 2 S: each super-tile's slice of the super list
    unsigned* cell_seg0;                           // S + 1: first segment of each super-tile
    unsigned *seg_cell, *seg_lo, *seg_hi;          // max_seg each
    unsigned *seg_cnt, *seg_base;                  // max_seg * kCellTiles each
    unsigned *tile_cnt, *tile_start;               // T each
    unsigned max_seg;
    int n_cells;                                   // S
};

// Super-tiles (cells) of 4 x 4 tiles; a cell's Gaussian list is expanded to
// its 16 tiles in segments of kSeg list entries.
constexpr int kSuper = 4;
constexpr int kCellTiles = kSuper * kSuper;
constexpr int kSeg = 1024;
static_assert(kCellTiles <= 32, "a cell's tile mask is one 32-bit word");

// The super-tile route serves images of at most 256 x 256 cells (1024 tiles
// a side); larger ones take the emit + radix-sort-by-tile-id route.
inline bool super_binning(int TX, int TY) {
    const int SX = (TX + kSuper - 1) / kSuper, SY = (TY + kSuper - 1) / kSuper;
    return SX <= (1 << kFusedMaxBits) && SY <= (1 << kFusedMaxBits);
}

size_t carve(void* base, int N, unsigned capacity, int TX, int TY, BinWs* w) {
    size_t off = sizeof(WsHeader);
    char* b = reinterpret_cast<char*>(base);
    auto take = [&](size_t bytes) -> void* {
        void* p = b ? b + off : nullptr;
        off += align_up(bytes, 256);
        return p;
    };
    const size_t n = (size_t)N, cap = (size_t)capacity;
    BinWs t;
    t.hdr = reinterpret_cast<WsHeader*>(base);
    t.misc = (SortMisc*)take(sizeof(SortMisc));
    t.dkeys0 = (unsigned*)take(n * 4);
    t.dvals0 = (unsigned*)take(n * 4);
    t.dkeys1 = (unsigned*)take(n * 4);
    t.dvals1 = (unsigned*)take(n * 4);
    t.pair_off = (unsigned*)take((n + 1) * 4);
    t.cnt_rank = (unsigned*)take(n * 4);
    t.scan_part = (unsigned*)take(((n + kScanTile - 1) / kScanTile + 1) * 4);
    t.tkeys0 = (unsigned*)take(cap * 4);
    t.tvals0 = (unsigned*)take(cap * 4);
    t.tkeys1 = (unsigned*)take(cap * 4);
    t.tvals1 = (unsigned*)take(cap * 4);
    t.hist = (unsigned*)take((size_t)kMaxPasses * kRadixMax * kSortMaxGrid * 4);
    t.totals = (unsigned*)take((size_t)kMaxPasses * kRadixMax * 4);
    t.gtot = (unsigned*)take((size_t)kMaxPasses * kMaxGroups * kRadixMax * 4);
    const bool sup = super_binning(TX, TY);
    const size_t S = sup ? (size_t)((TX + kSuper - 1) / kSuper) * ((TY + kSuper - 1) / kSuper) : 0;
    const size_t T = sup ? (size_t)TX * TY : 0;
    t.max_seg = sup ? (unsigned)(cap / kSeg + S + 1) : 0u;
    t.n_cells = (int)S;
    const size_t ms = t.max_seg;
    t.rc_rank = (unsigned*)take(sup ? n * 4 : 0);
    t.sub_rank = (unsigned char*)take(sup ? n : 0);
    t.owner_lo = (unsigned*)take((size_t)kSortMaxGrid * 4);
    t.owner_hi = (unsigned*)take((size_t)kSortMaxGrid * 4);
    t.cell_ranges = (unsigned*)take(2 * S * 4);
    t.cell_seg0 = (unsigned*)take((S + 1) * 4);
    t.seg_cell = (unsigned*)take(ms * 4);
    t.seg_lo = (unsigned*)take(ms * 4);
    t.seg_hi = (unsigned*)take(ms * 4);
    t.seg_cnt = (unsigned*)take(ms * kCellTiles * 4);
    t.seg_base = (unsigned*)take(ms * kCellTiles * 4);
    t.tile_cnt = (unsigned*)take(T * 4);
    t.tile_start = (unsigned*)take(T * 4);
    if (w) *w = t;
    return off;
}

// A visible Gaussian's rectangle of super-tiles in 32 bits (x0, y0 < 256;
// width and height in 1..256): x0 | (w - 1) << 8 | y0 << 16 | (h - 1) << 24.
__device__ __forceinline__ int4 super_rect(int4 rc) {
    return make_int4(rc.x / kSuper, rc.y / kSuper, (rc.z - 1) / kSuper + 1, (rc.w - 1) / kSuper + 1);
}
__device__ __forceinline__ unsigned pack_rect(int4 rc) {
    return (unsigned)rc.x | ((unsigned)(rc.z - rc.x - 1) << 8) | ((unsigned)rc.y << 16) |
           ((unsigned)(rc.w - rc.y - 1) << 24);
}
__device__ __forceinline__ int rect_x0(unsigned p) { return (int)(p & 255u); }
__device__ __forceinline__ int rect_w(unsigned p) { return (int)((p >> 8) & 255u) + 1; }
__device__ __forceinline__ int rect_y0(unsigned p) { return (int)((p >> 16) & 255u); }
__device__ __forceinline__ int rect_h(unsigned p) { return (int)(p >> 24) + 1; }

// Where a Gaussian's tile rectangle starts and ends inside the first and
// last cells of its cell rectangle, in 8 bits: x0 mod 4 | (x1 - 1) mod 4 << 2
// | y0 mod 4 << 4 | (y1 - 1) mod 4 << 6 (tile rectangle [x0, x1) x [y0, y1)).
__device__ __forceinline__ unsigned sub_offsets(int4 rc) {
    static_assert(kSuper == 4, "two bits per offset assume 4 x 4 cells");
    return (unsigned)(rc.x & 3) | (unsigned)((rc.z - 1) & 3) << 2 | (unsigned)(rc.y & 3) << 4 |
           (unsigned)((rc.w - 1) & 3) << 6;
}

// Cell-pair keys: cell x in bits 0-7 and cell y in bits 16-23 (the radix
// digits), the 16-bit mask of the cell's tiles that the Gaussian covers in
// bits 8-15 (mask bits 0-7) and 24-31 (mask bits 8-15); bit ly * 4 + lx of
// the mask is tile (4 cy + ly, 4 cx + lx).
constexpr unsigned kCellBits = 0x00FF00FFu;
__device__ __forceinline__ unsigned key_mask(unsigned key) { return ((key >> 8) & 0xFFu) | ((key >> 24) << 8); }

// The key of the pair (cell (cx, cy), Gaussian) from the Gaussian's packed
// cell rectangle rc and sub_offsets byte sb: the tiles covered span lx0..lx1
// in x (the rectangle's offsets in its first / last cell column, else 0 / 3)
// and ly0..ly1 in y.
__device__ __forceinline__ unsigned cell_pair_key(unsigned rc, unsigned sb, int cx, int cy) {
    const int cx0 = rect_x0(rc), cy0 = rect_y0(rc);
    const unsigned lx0 = cx == cx0 ? (sb & 3u) : 0u;
    const unsigned lx1 = cx == cx0 + rect_w(rc) - 1 ? ((sb >> 2) & 3u) : 3u;
    const unsigned ly0 = cy == cy0 ? ((sb >> 4) & 3u) : 0u;
    const unsigned ly1 = cy == cy0 + rect_h(rc) - 1 ? (sb >> 6) : 3u;
    const unsigned row = ((2u << lx1) - (1u << lx0)) * 0x1111u;  // tiles lx0..lx1 of every row
    const unsigned rows = (2u << (4u * ly1 + 3u)) - (1u << (4u * ly0));  // rows ly0..ly1
    const unsigned m = row & rows;
    return (unsigned)cx | (m & 0xFFu) << 8 | (unsigned)cy << 16 | (m >> 8) << 24;
}

// Debug build: after a failed index check inside the binning, later kernels
// would see inconsistent inputs (a visible rank without pairs, an unwritten
// pair), so the frame's usable pair count is set to 0: every later kernel of
// the call then sees an empty frame (all ranges empty, no pair written), as
// when the capacity is exceeded.
__device__ __forceinline__ void abort_frame(SortMisc* misc) { atomicExch(&misc->p_eff, 0u); }

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Zero the ranges and the per-pass digit totals, build the depth keys, check
// the pair count against the capacity.
__global__ void k_bin_init(int N, int T, const float* __restrict__ depth, const unsigned* __restrict__ tiles_touched,
                           const unsigned* __restrict__ d_num_pairs, unsigned capacity, BinWs w,
                           unsigned* __restrict__ ranges) {
    pdl_enter();
    const int stride = gridDim.x * blockDim.x;
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = tid; i < 2 * T; i += stride) ranges[i] = 0u;
    for (int i = tid; i < kMaxPasses * kRadixMax; i += stride) w.totals[i] = 0u;
    for (int i = tid; i < kMaxPasses * kMaxGroups * kRadixMax; i += stride) w.gtot[i] = 0u;
    // cell ranges [start, end) are found by atomic min / max in the last
    // cell pass: starts from above, ends from below (empty: start > end)
    for (int i = tid; i < 2 * w.n_cells; i += stride) w.cell_ranges[i] = (i & 1) ? 0u : 0xFFFFFFFFu;
    // four items per thread and round, their loads issued together
    constexpr int kU = 4;
    for (long long i0 = tid; i0 < N; i0 += (long long)kU * stride) {
        unsigned tt[kU], dk[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const long long i = i0 + (long long)u * stride;
            tt[u] = i < N ? tiles_touched[i] : 0u;
            dk[u] = i < N ? __float_as_uint(depth[i]) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const long long i = i0 + (long long)u * stride;
            if (i < N) {
                w.dkeys0[i] = tt[u] > 0 ? dk[u] : 0xFFFFFFFFu;
                w.dvals0[i] = (unsigned)i;
            }
        }
    }
    if (tid == 0) {
        const unsigned P = *d_num_pairs;
        w.misc->n_gauss = (unsigned)N;
        if (P > capacity) {
            raise_status(w.hdr, GS_ERR_CAPACITY);
            w.misc->p_eff = 0;
        } else {
            w.misc->p_eff = P;
        }
    }
}

// Radix passes.  A pass over n keys runs on G CTAs, each owning one
// contiguous chunk of the input (a multiple of its tile of ITEMS x 256
// keys), so that equal digits keep their input order: chunk, then tile,
// then item slot j, then warp, then lane.  MAXB is the widest digit the
// kernel instance handles; `bits` <= MAXB is the width of this pass.
template <int MAXB>
struct RadixCfg {
    static constexpr int kRadix = 1 << MAXB;
    static constexpr int kItems = 8;                        // keys per thread per tile
    static constexpr int kTileKeys = kItems * kSortBlock;   // 2048
    static constexpr int kWarps = kSortBlock / 32;
    static constexpr int kWarpKeys = kItems * 32;           // each warp owns a contiguous block of the tile
    // scatter shared memory: per-digit running bases / tile counts / tile
    // starts / tile bases, per-(warp, digit) counts turned into offsets, and
    // the tile's keys and values regrouped by digit
    static constexpr size_t kScatterSmem = (size_t)(4 * kRadix + kWarps * kRadix + 2 * kTileKeys) * sizeof(unsigned);
};

// Keys per CTA of a pass over n keys on G CTAs: ceil(n / G) rounded up to
// whole 2048-key tiles (the same for every digit width).
__host__ __device__ __forceinline__ unsigned chunk_size(unsigned n, unsigned G) {
    constexpr unsigned tile = 2048;
    const unsigned long long c = ((unsigned long long)n + G - 1) / G;
    return (unsigned)((c + tile - 1) / tile * tile);
}

template <int MAXB>
__device__ __forceinline__ void chunk_of(unsigned n, unsigned& lo, unsigned& hi) {
    static_assert(RadixCfg<MAXB>::kTileKeys == 2048, "chunk_size assumes 2048-key tiles");
    const unsigned chunk = chunk_size(n, gridDim.x);
    const unsigned long long l = (unsigned long long)blockIdx.x * chunk;
    lo = l < n ? (unsigned)l : n;
    hi = (unsigned)min((unsigned long long)n, (unsigned long long)lo + chunk);
}

constexpr unsigned kNoDigit = 0xFFFFFFFFu;

// Lanes of the warp holding the same digit as this lane, from one ballot per
// digit bit (a warp-level multi-split); lanes without a key form their own
// group.  Cheaper than __match_any_sync, whose throughput limited the passes.
template <int MAXB>
__device__ __forceinline__ unsigned digit_peers(unsigned d, int bits) {
    const bool valid = d != kNoDigit;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    unsigned m = valid ? vmask : ~vmask;
#pragma unroll
    for (int b = 0; b < MAXB; ++b) {
        if (b < bits) {
            const bool bit = (d >> b) & 1u;
            const unsigned v = __ballot_sync(0xffffffffu, bit);
            m &= bit ? v : ~v;
        }
    }
    return m;
}

// Per-CTA digit histogram of its chunk, stored chunk-major
// (hist[cta * kRadixMax + d]); digit totals accumulate into totals[d] and the
// totals of each group of kScanGroup consecutive chunks into
// gtot[group * kRadixMax + d] (see chunk_bases).  Each warp counts into its
// own shared-memory histogram.
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock)
k_radix_hist(const unsigned* __restrict__ keys, const unsigned* __restrict__ n_ptr, int shift, int bits,
             unsigned* __restrict__ hist, unsigned* __restrict__ totals, unsigned* __restrict__ gtot) {
    pdl_enter();
    using C = RadixCfg<MAXB>;
    __shared__ unsigned s_h[C::kWarps][C::kRadix];
    const int radix = 1 << bits;
    const unsigned mask = radix - 1;
    for (int i = threadIdx.x; i < C::kWarps * C::kRadix; i += kSortBlock) (&s_h[0][0])[i] = 0;
    __syncthreads();
    unsigned lo, hi;
    chunk_of<MAXB>(*n_ptr, lo, hi);
    const int warp = threadIdx.x >> 5;
    // chunk boundaries are multiples of the tile (2048 keys), so every tile
    // but the last is read with 16-byte loads, 4 keys per load
    for (unsigned base = lo; base < hi; base += C::kTileKeys) {
        if (base + C::kTileKeys <= hi) {
            const uint4* k4 = reinterpret_cast<const uint4*>(keys + base);
            uint4 v[C::kItems / 4];
#pragma unroll
            for (int j = 0; j < C::kItems / 4; ++j) v[j] = k4[j * kSortBlock + threadIdx.x];
#pragma unroll
            for (int j = 0; j < C::kItems / 4; ++j) {
                atomicAdd(&s_h[warp][(v[j].x >> shift) & mask], 1u);
                atomicAdd(&s_h[warp][(v[j].y >> shift) & mask], 1u);
                atomicAdd(&s_h[warp][(v[j].z >> shift) & mask], 1u);
                atomicAdd(&s_h[warp][(v[j].w >> shift) & mask], 1u);
            }
        } else {
            for (unsigned i = base + threadIdx.x; i < hi; i += kSortBlock)
                atomicAdd(&s_h[warp][(keys[i] >> shift) & mask], 1u);
        }
    }
    __syncthreads();
    for (int dd = threadIdx.x; dd < radix; dd += kSortBlock) {
        unsigned c = 0;
#pragma unroll
        for (int w = 0; w < C::kWarps; ++w) c += s_h[w][dd];
        hist[(size_t)blockIdx.x * kRadixMax + dd] = c;
        if (c) {
            atomicAdd(&totals[dd], c);
            atomicAdd(&gtot[(blockIdx.x / kScanGroup) * kRadixMax + dd], c);
        }
    }
}

// Global output base of each digit for this CTA's chunk (thread d < radix
// writes base[d]): the totals of the smaller digits, plus digit d's counts in
// the chunks before this one - whole groups of kScanGroup chunks from the
// group totals, the rest of this chunk's group from the chunk counts.  At
// most kMaxGroups - 1 + kScanGroup - 1 independent loads per thread, each a
// coalesced row over the digits; no separate scan pass over the histograms.
// Ends with a block barrier.
__device__ __forceinline__ void chunk_bases(const unsigned* __restrict__ hist, const unsigned* __restrict__ totals,
                                            const unsigned* __restrict__ gtot, int radix, unsigned* __restrict__ base) {
    static_assert(kSortBlock == kRadixMax, "one thread per digit");
    __shared__ unsigned s_w[kSortBlock / 32 + 1];
    const int d = threadIdx.x;
    const unsigned c = blockIdx.x, g = c / kScanGroup;
    const bool in = d < radix;
    const unsigned t = in ? totals[d] : 0u;
    unsigned pre = 0;
    if (in) {
#pragma unroll
        for (int k = 0; k < kMaxGroups - 1; ++k)
            if ((unsigned)k < g) pre += gtot[k * kRadixMax + d];
#pragma unroll
        for (int k = 0; k < kScanGroup - 1; ++k) {
            const unsigned cc = g * kScanGroup + (unsigned)k;
            if (cc < c) pre += hist[(size_t)cc * kRadixMax + d];
        }
    }
    // exclusive prefix of the digit totals over the block
    const int lane = d & 31, warp = d >> 5;
    unsigned incl = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    unsigned wbase = 0;
#pragma unroll
    for (int k = 0; k < kSortBlock / 32; ++k)
        if (k < warp) wbase += s_w[k];
    if (in) base[d] = wbase + incl - t + pre;
    __syncthreads();
}

// Stable scatter of one tile of up to 2048 keys, each warp owning a
// contiguous block of 256 of them (8 rows of 32), keys and digits already in
// registers (row j of warp w = tile positions w*256 + j*32 + lane):
//   1. each warp ranks its keys row by row (digit_peers within the row, plus
//      a running per-digit count of the warp's earlier rows), so ranks follow
//      input order within the warp;
//   2. one thread per digit turns the warps' counts into offsets (warp
//      order), giving the tile's count per digit; one warp scans those into
//      tile-local digit starts and advances the running global bases;
//   3. every key is placed in shared memory at its tile-local sorted position;
//   4. the regrouped tile is written out in order, so consecutive lanes write
//      consecutive addresses of one digit's run (coalesced stores); with
//      cell_ranges (the last cell pass), the first and last key of each local
//      run of one cell extend that cell's range by an atomic min / max.
// keys_out may be null (values only).  Ends with a block barrier.
template <int MAXB>
struct ScatterSmem {
    using C = RadixCfg<MAXB>;
    unsigned* base;   // [radix] running global base
    unsigned* tcnt;   // [radix] this tile's count per digit
    unsigned* tstart; // [radix] tile-local start per digit
    unsigned* tdelta; // [radix] global base for this tile minus the tile-local start (mod 2^32)
    unsigned* wcnt;   // [warps][radix] counts, then offsets
    unsigned* keys;   // [tile (+ padding)] regrouped keys
    unsigned* vals;   // [tile (+ padding)] regrouped values
    __device__ ScatterSmem(unsigned char* raw, size_t tile_words) {
        base = reinterpret_cast<unsigned*>(raw);
        tcnt = base + C::kRadix;
        tstart = tcnt + C::kRadix;
        tdelta = tstart + C::kRadix;
        wcnt = tdelta + C::kRadix;
        keys = wcnt + C::kWarps * C::kRadix;
        vals = keys + tile_words;
    }
    static constexpr size_t bytes(size_t tile_words) {
        return (size_t)(4 * C::kRadix + C::kWarps * C::kRadix) * sizeof(unsigned) + 2 * tile_words * sizeof(unsigned);
    }
};

template <int MAXB>
__device__ __forceinline__ void scatter_tile(const ScatterSmem<MAXB>& sm, const unsigned (&key)[RadixCfg<MAXB>::kItems],
                                             const unsigned (&val)[RadixCfg<MAXB>::kItems],
                                             const unsigned (&d)[RadixCfg<MAXB>::kItems], unsigned tile_n, int shift,
                                             int bits, unsigned* __restrict__ keys_out,
                                             unsigned* __restrict__ vals_out, unsigned* __restrict__ cell_ranges,
                                             int SX) {
    using C = RadixCfg<MAXB>;
    const int radix = 1 << bits;
    const unsigned mask = radix - 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
    unsigned* wcnt = sm.wcnt + warp * C::kRadix;
    unsigned rank[C::kItems];
    for (int dd = lane; dd < radix; dd += 32) wcnt[dd] = 0;
    __syncwarp();
    // 1. ranks within the warp, row after row
#pragma unroll
    for (int j = 0; j < C::kItems; ++j) {
        const unsigned peers = digit_peers<MAXB>(d[j], bits);
        const bool valid = d[j] != kNoDigit;
        const unsigned before = valid ? wcnt[d[j]] : 0u;
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) wcnt[d[j]] = before + __popc(peers);
        __syncwarp();
        rank[j] = before + __popc(peers & lt);
    }
    __syncthreads();
    // 2. per digit: warp offsets in warp order, and the tile count
    for (int dd = threadIdx.x; dd < radix; dd += kSortBlock) {
        unsigned run = 0;
#pragma unroll
        for (int w = 0; w < C::kWarps; ++w) {
            const unsigned c = sm.wcnt[w * C::kRadix + dd];
            sm.wcnt[w * C::kRadix + dd] = run;
            run += c;
        }
        sm.tcnt[dd] = run;
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int per = (C::kRadix + 31) / 32;
        unsigned v[per], sum = 0;
#pragma unroll
        for (int k = 0; k < per; ++k) {
            const int dd = lane * per + k;
            v[k] = dd < radix ? sm.tcnt[dd] : 0u;
            sum += v[k];
        }
        unsigned incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        unsigned run = incl - sum;
#pragma unroll
        for (int k = 0; k < per; ++k) {
            const int dd = lane * per + k;
            if (dd < radix) {
                sm.tstart[dd] = run;
                sm.tdelta[dd] = sm.base[dd] - run;
                sm.base[dd] += v[k];
            }
            run += v[k];
        }
    }
    __syncthreads();
    // 3. regroup the tile by digit in shared memory
#pragma unroll
    for (int j = 0; j < C::kItems; ++j) {
        if (d[j] != kNoDigit) {
            const unsigned loc = sm.tstart[d[j]] + wcnt[d[j]] + rank[j];
            sm.keys[loc] = key[j];
            sm.vals[loc] = val[j];
        }
    }
    __syncthreads();
    // 4. write the regrouped tile: consecutive q of one digit go to
    //    consecutive output positions
    for (unsigned q = threadIdx.x; q < tile_n; q += kSortBlock) {
        const unsigned k2 = sm.keys[q];
        const unsigned dq = (k2 >> shift) & mask;
        const unsigned pos = q + sm.tdelta[dq];
        if (keys_out) keys_out[pos] = k2;
        vals_out[pos] = sm.vals[q];
        if (cell_ranges) {
            // last cell pass: within its digit's run the tile is in cell
            // order, so a cell's keys from this tile are one local run; the
            // first and last keys of each run extend the cell's range
            const unsigned r0 = sm.tstart[dq], r1 = r0 + sm.tcnt[dq];
            const bool first = q == r0 || ((sm.keys[q - 1] ^ k2) & kCellBits) != 0u;
            const bool last = q + 1 == r1 || ((sm.keys[q + 1] ^ k2) & kCellBits) != 0u;
            if (first || last) {
                const unsigned c = ((k2 >> 16) & 0xFFu) * (unsigned)SX + (k2 & 0xFFu);
                if (first) atomicMin(&cell_ranges[2 * c], pos);
                if (last) atomicMax(&cell_ranges[2 * c + 1], pos + 1);
            }
        }
    }
    __syncthreads();  // the next tile reuses every shared array
}

// Stable scatter pass over keys in global memory: each CTA walks its chunk
// tile by tile.
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock)
k_radix_scatter(const unsigned* __restrict__ keys_in, const unsigned* __restrict__ vals_in,
                unsigned* __restrict__ keys_out, unsigned* __restrict__ vals_out,
                const unsigned* __restrict__ n_ptr, int shift, int bits, const unsigned* __restrict__ hist,
                const unsigned* __restrict__ totals, const unsigned* __restrict__ gtot,
                unsigned* __restrict__ cell_ranges, int SX) {
    pdl_enter();
    using C = RadixCfg<MAXB>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const ScatterSmem<MAXB> sm(smem_raw, C::kTileKeys);
    const int radix = 1 << bits;
    const unsigned mask = radix - 1;
    chunk_bases(hist, totals, gtot, radix, sm.base);
    unsigned lo, hi;
    chunk_of<MAXB>(*n_ptr, lo, hi);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (unsigned base = lo; base < hi; base += C::kTileKeys) {
        const unsigned tile_n = min((unsigned)C::kTileKeys, hi - base);
        unsigned key[C::kItems], val[C::kItems], d[C::kItems];
        const unsigned wbase = base + warp * C::kWarpKeys;
#pragma unroll
        for (int j = 0; j < C::kItems; ++j) {
            const unsigned i = wbase + j * 32 + lane;
            const bool valid = i < hi;
            key[j] = valid ? keys_in[i] : 0u;
            val[j] = valid ? vals_in[i] : 0u;
            d[j] = valid ? (key[j] >> shift) & mask : kNoDigit;
        }
        scatter_tile<MAXB>(sm, key, val, d, tile_n, shift, bits, keys_out, vals_out, cell_ranges, SX);
    }
}

// Exclusive scan, in depth-rank order, of the pair counts:
// pair_off[r] = sum over ranks r' < r of cnt_rank[r'], where cnt_rank[r] is
// the number of tiles of Gaussian order[r] or, with `rect` (super-tile
// route), of its cells.  The first kernel gathers each rank's count once
// (and, on the super-tile route, its packed cell rectangle).
__global__ void __launch_bounds__(kSortBlock)
k_scan_partials(int N, const unsigned* __restrict__ order, const unsigned* __restrict__ tiles_touched,
                const int4* __restrict__ rect, unsigned* __restrict__ cnt_rank, unsigned* __restrict__ rc_rank,
                unsigned char* __restrict__ sub_rank,
                unsigned* __restrict__ part, SortMisc* __restrict__ misc) {
    pdl_enter();
    const int base = blockIdx.x * kScanTile;
    // the gathers are issued in two rounds of independent loads (all ids,
    // then every count and rectangle), not as one dependent chain per rank
    unsigned g[kScanItems];
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k * kSortBlock + threadIdx.x;
        g[k] = r < N ? order[r] : 0xFFFFFFFFu;
    }
    unsigned v[kScanItems];
    int4 tr[kScanItems];
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const bool ok = g[k] < (unsigned)N && id_ok(g[k]);
        v[k] = ok ? tiles_touched[g[k]] : 0u;
        if (rect) tr[k] = ok ? rect[g[k]] : make_int4(0, 0, 0, 0);
    }
    unsigned s = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k * kSortBlock + threadIdx.x;
        if (r < N) {
            if (!id_ok(g[k])) abort_frame(misc);
            unsigned c = v[k];
            if (rect && c) {
                const int4 sr = super_rect(tr[k]);
                c = (unsigned)((sr.z - sr.x) * (sr.w - sr.y));
                rc_rank[r] = pack_rect(sr);
                sub_rank[r] = (unsigned char)sub_offsets(tr[k]);
            }
            cnt_rank[r] = c;
            s += c;
        }
    }
    s = __reduce_add_sync(0xffffffffu, s);
    __shared__ unsigned s_w[kSortBlock / 32];
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned t = 0;
        for (int k = 0; k < kSortBlock / 32; ++k) t += s_w[k];
        part[blockIdx.x] = t;
    }
}

// Second half of the rank-order scan: each CTA takes the exclusive prefix of
// the first kernel's per-CTA sums below it and the grand total (the frame's
// pairs - of super-tile pairs on the super-tile route - stored by CTA 0 in
// misc->ps, or 0 if the frame's pairs exceed the capacity) from the sums
// directly (at most a few loads per thread), then scans its own ranks.
// With `owner_lo` (super-tile route, G CTAs per pair pass), also records for
// every chunk c of the pair stream the rank owning its first pair
// (owner_lo[c]) and its last pair (owner_hi[c]): each rank checks the chunk
// boundaries inside its own pair range, so no search is needed later.
__global__ void __launch_bounds__(kSortBlock)
k_scan_down(int N, const unsigned* __restrict__ cnt_rank, const unsigned* __restrict__ part,
            unsigned* __restrict__ pair_off, SortMisc* __restrict__ misc, unsigned G,
            unsigned* __restrict__ owner_lo, unsigned* __restrict__ owner_hi) {
    pdl_enter();
    __shared__ unsigned s_pre[kSortBlock / 32], s_tot[kSortBlock / 32];
    unsigned pre = 0, tot = 0;
    constexpr int kP = 8;  // partial sums per thread and round, loaded together
    for (unsigned i0 = 0; i0 < gridDim.x; i0 += kP * kSortBlock) {
        unsigned pv[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            const unsigned i = i0 + k * kSortBlock + threadIdx.x;
            pv[k] = i < gridDim.x ? part[i] : 0u;
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            tot += pv[k];
            if (i0 + k * kSortBlock + threadIdx.x < blockIdx.x) pre += pv[k];
        }
    }
    pre = __reduce_add_sync(0xffffffffu, pre);
    tot = __reduce_add_sync(0xffffffffu, tot);
    // each thread owns kScanItems consecutive ranks
    const int base = blockIdx.x * kScanTile + threadIdx.x * kScanItems;
    unsigned v[kScanItems];
    unsigned local = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k;
        v[k] = r < N ? cnt_rank[r] : 0u;
        local += v[k];
    }
    __shared__ unsigned s_w[kSortBlock / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_w[warp] = incl;
    if (lane == 0) {
        s_pre[warp] = pre;
        s_tot[warp] = tot;
    }
    __syncthreads();
    unsigned cta_pre = 0, total = 0;
#pragma unroll
    for (int k = 0; k < kSortBlock / 32; ++k) {
        cta_pre += s_pre[k];
        total += s_tot[k];
    }
    const unsigned ps = misc->p_eff ? total : 0u;
    if (blockIdx.x == 0 && threadIdx.x == 0) misc->ps = ps;
    unsigned wbase = 0;
    for (int k = 0; k < warp; ++k) wbase += s_w[k];
    unsigned run = cta_pre + wbase + incl - local;
    const unsigned P = owner_lo ? ps : 0u;
    const unsigned long long chunk = P ? chunk_size(P, G) : 1ull;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k;
        if (r < N) pair_off[r] = run;
        if (P && v[k] && r < N) {
            const unsigned long long off = run, e = off + v[k];
            for (unsigned long long c = off / chunk; c * chunk < e && c < G; ++c) {
                if (c * chunk >= off) owner_lo[c] = (unsigned)r;
                const unsigned long long last = min((c + 1) * chunk, (unsigned long long)P) - 1;
                if (last >= off && last < e) owner_hi[c] = (unsigned)r;
            }
        }
        run += v[k];
    }
}

// Emit the (tile, Gaussian) pairs in depth-rank order, balanced by pairs:
// CTA c writes output positions [c * 2048, (c + 1) * 2048).  Visible
// Gaussians come first in rank order and each has at least one pair, so
// the ranks covering a segment are found by one binary search over the
// exclusive pair offsets and number at most 2049; their offsets and ids are
// staged in shared memory, and each thread finds the owner of each of its
// output positions by a binary search there.  Row and column within the
// Gaussian's tile rectangle come from a float quotient corrected by one step
// (local < 2^24 and width <= 4096, so the float error is below one).
constexpr int kEmitSeg = 2048;

__device__ __forceinline__ unsigned upper_bound_global(const unsigned* __restrict__ a, unsigned n, unsigned x) {
    // first index i in [0, n) with a[i] > x (n if none)
    unsigned lo = 0, hi = n;
    while (lo < hi) {
        const unsigned mid = (lo + hi) >> 1;
        if (a[mid] <= x) lo = mid + 1; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kSortBlock)
k_emit(int N, int TX, const unsigned* __restrict__ order, const unsigned* __restrict__ pair_off,
       const int4* __restrict__ rect, const unsigned* __restrict__ tiles_touched, SortMisc* __restrict__ misc,
       unsigned* __restrict__ tkeys, unsigned* __restrict__ tvals) {
    pdl_enter();
    __shared__ unsigned s_off[kEmitSeg + 1];
    __shared__ unsigned s_g[kEmitSeg + 1];
    __shared__ unsigned s_r0, s_nr;
    const unsigned P = misc->p_eff;
    if (P == 0) return;  // nothing to emit, or over capacity
    for (unsigned p0 = blockIdx.x * kEmitSeg; p0 < P; p0 += gridDim.x * kEmitSeg) {
        const unsigned p1 = min(P, p0 + kEmitSeg);
        __syncthreads();  // the previous segment's readers are done
        if (threadIdx.x == 0) {
            // ranks r0 .. r1-1 cover [p0, p1): r0 = last rank with offset <= p0
            const unsigned r0 = upper_bound_global(pair_off, (unsigned)N, p0) - 1;
            const unsigned r1 = upper_bound_global(pair_off, (unsigned)N, p1 - 1);
            s_r0 = r0;
            s_nr = min(r1 - r0, (unsigned)kEmitSeg + 1);
        }
        __syncthreads();
        const unsigned r0 = s_r0, nr = s_nr;
        for (unsigned i = threadIdx.x; i < nr; i += kSortBlock) {
            s_off[i] = pair_off[r0 + i];
            s_g[i] = order[r0 + i];
        }
        __syncthreads();
        for (unsigned p = p0 + threadIdx.x; p < p1; p += kSortBlock) {
            // owner: last staged rank whose offset <= p
            unsigned lo = 0, hi = nr;
            while (hi - lo > 1) {
                const unsigned mid = (lo + hi) >> 1;
                if (s_off[mid] <= p) lo = mid; else hi = mid;
            }
            const unsigned g = s_g[lo];
            if (!id_ok(g) || !pos_ok(p)) {
                abort_frame(misc);
                continue;
            }
            const int4 rc = rect[g];
            const unsigned w = (unsigned)(rc.z - rc.x);
            const unsigned local = p - s_off[lo];
            unsigned q = (unsigned)__fdividef((float)local, (float)w);
            int r = (int)local - (int)(q * w);
            if (r < 0) { --q; r += (int)w; }
            else if (r >= (int)w) { ++q; r -= (int)w; }
            tkeys[p] = (unsigned)(rc.y + (int)q) * (unsigned)TX + (unsigned)(rc.x + r);
            tvals[p] = g;
        }
    }
}

// ranges[t] = [first, last + 1) of tile t in the sorted list, found by
// comparing neighbours; four keys per thread with 16-byte loads, neighbours
// across lanes by shuffles.  Optional 64-bit keys for callers that want them.
__global__ void k_ranges(const unsigned* __restrict__ tkeys, const unsigned* __restrict__ ids,
                         const float* __restrict__ depth, const SortMisc* __restrict__ misc, unsigned* __restrict__ ranges,
                         unsigned long long* __restrict__ keys) {
    pdl_enter();
    const unsigned P = misc->p_eff;
    const unsigned nq = (P + 3) / 4;  // quads, the last one partial
    const unsigned stride = gridDim.x * blockDim.x;
    const int lane = threadIdx.x & 31;
    // every lane of a warp iterates the same number of times (shuffles below)
    for (unsigned qb = blockIdx.x * blockDim.x + (threadIdx.x & ~31u); qb < nq; qb += stride) {
        const unsigned qi = qb + lane;
        const unsigned k0 = qi * 4;
        unsigned t[4];
        if (k0 + 3 < P) {
            const uint4 v = reinterpret_cast<const uint4*>(tkeys)[qi];
            t[0] = v.x; t[1] = v.y; t[2] = v.z; t[3] = v.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) t[j] = k0 + j < P ? tkeys[k0 + j] : 0xFFFFFFFFu;
        }
        unsigned prev = __shfl_up_sync(0xffffffffu, t[3], 1);
        unsigned next = __shfl_down_sync(0xffffffffu, t[0], 1);
        if (lane == 0) prev = (k0 > 0 && k0 - 1 < P) ? tkeys[k0 - 1] : 0xFFFFFFFFu;
        if (lane == 31) next = (k0 + 4 < P) ? tkeys[k0 + 4] : 0xFFFFFFFFu;
        if (qi < nq) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const unsigned k = k0 + j;
                if (k >= P) break;
                const unsigned before = j == 0 ? prev : t[j - 1];
                const unsigned after = (j == 3 || k + 1 == P) ? (k + 1 == P ? 0xFFFFFFFFu : next) : t[j + 1];
                if (k == 0 || before != t[j]) ranges[2 * t[j]] = k;
                if (k + 1 == P || after != t[j]) ranges[2 * t[j] + 1] = k + 1;
                if (keys && pos_ok(k) && id_ok(ids[k]))
                    keys[k] = ((unsigned long long)t[j] << 32) | __float_as_uint(depth[ids[k]]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Super-tile binning (images of at most 256 x 256 cells of 4 x 4 tiles).
// Most pairs come from Gaussians that cover many tiles, so instead
// of sorting every (tile, Gaussian) pair, the Gaussians are first binned to
// super-tiles (cells), which yields far fewer pairs, and each super-tile's
// depth-ordered Gaussian list is then expanded to its 16 tiles directly into
// the final per-tile lists:
//   1. cell binning: the (cell, Gaussian) pairs of the rank-order stream are
//      stably sorted by cell; the cell order cy * SX + cx equals the
//      lexicographic (cy, cx) order, so this is a stable pass on cx followed
//      by a stable pass on cy.  The first pass does not read a materialised
//      pair list: it generates the pairs of its chunk of the stream on the
//      fly (Gaussian by Gaussian, each cell rectangle row-major) and ranks
//      them by cx; its histogram comes from the cell rectangles directly (a
//      difference array over cx).  Intermediate key: cx | cy << 16, with
//      the pair's 16-bit tile mask in the other bits (cell_pair_key), so
//      that later steps never look the Gaussian's rectangle up again.
//   2. each cell's list is cut into segments of kSeg entries; per segment and
//      tile of the cell, the number of its Gaussians touching the tile
//      (warp ballots over the 16-bit tile masks);
//   3. prefix sums give every tile's range and every (segment, tile) base;
//   4. each segment writes its Gaussians into the tiles' lists: for every
//      tile bit, a ballot ranks the warp's Gaussians touching that tile, so
//      consecutive lanes write consecutive positions.
// Within a tile the order is the cell list's order, which is rank order, so
// the result is the (tile, depth, id) order.
constexpr int kGenWin = 9 * kSortBlock;   // staged ranks per 2048-pair tile (at most 2049 needed)
constexpr int kPadTile = RadixCfg<8>::kTileKeys + RadixCfg<8>::kTileKeys / 32;

// Padded shared-memory index: one spare word per 32, so that thread t's
// consecutive slots 8t .. 8t+7 and a warp's row of 32 are both free of bank
// conflicts.
__device__ __forceinline__ unsigned pad_idx(unsigned q) { return q + (q >> 5); }

// Per-CTA x histogram of the CTA's chunk of the cell-pair stream (the chunk that
// k_gen_scatter will rank).  Gaussians entirely inside the chunk add their
// height to tx in [x0, x0 + w) through a difference array; the (at most two)
// Gaussians cut by the chunk's ends are counted pair by pair.
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock)
k_gen_hist(const unsigned* __restrict__ pair_off, const unsigned* __restrict__ rc_rank,
           const unsigned* __restrict__ n_ptr, const unsigned* __restrict__ owner_lo,
           const unsigned* __restrict__ owner_hi, unsigned* __restrict__ hist, unsigned* __restrict__ totals,
           unsigned* __restrict__ gtot) {
    pdl_enter();
    using C = RadixCfg<MAXB>;
    constexpr int kU = 4;  // ranks per thread in flight
    __shared__ int s_d[C::kRadix + 1];
    const unsigned P = *n_ptr;
    for (int i = threadIdx.x; i <= C::kRadix; i += kSortBlock) s_d[i] = 0;
    unsigned lo, hi;
    chunk_of<MAXB>(P, lo, hi);
    __syncthreads();
    if (lo < hi) {
        const unsigned ra = owner_lo[blockIdx.x], rb = owner_hi[blockIdx.x];
        for (unsigned rbase = ra; rbase <= rb; rbase += kU * kSortBlock) {
            unsigned off[kU], rc[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const unsigned r = rbase + u * kSortBlock + threadIdx.x;
                const bool ok = r <= rb;
                off[u] = ok ? pair_off[r] : 0xFFFFFFFFu;
                rc[u] = ok ? rc_rank[r] : 0u;
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                if (off[u] == 0xFFFFFFFFu) continue;
                const int x0 = rect_x0(rc[u]), w = rect_w(rc[u]), h = rect_h(rc[u]);
                const unsigned n = (unsigned)(w * h);
                if (off[u] >= lo && off[u] + n <= hi) {
                    atomicAdd(&s_d[x0], h);
                    atomicAdd(&s_d[x0 + w], -h);
                }
            }
        }
        // the cut Gaussians, pair by pair, by the whole CTA
        for (int e = 0; e < 2; ++e) {
            const unsigned r = e == 0 ? ra : rb;
            if (e == 1 && rb == ra) break;
            const unsigned rc = rc_rank[r];
            const unsigned off = pair_off[r];
            const unsigned w = (unsigned)rect_w(rc);
            const unsigned n = w * (unsigned)rect_h(rc);
            if (off >= lo && off + n <= hi) continue;  // not cut: counted above
            const unsigned a = max(off, lo) - off, b = min(off + n, hi) - off;
            for (unsigned l = a + threadIdx.x; l < b; l += kSortBlock) {
                const int tx = rect_x0(rc) + (int)(l % w);
                atomicAdd(&s_d[tx], 1);
                atomicAdd(&s_d[tx + 1], -1);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        // inclusive prefix of the difference array: the count per digit
        const int lane = threadIdx.x;
        constexpr int per = C::kRadix / 32;
        int v[per], sum = 0;
#pragma unroll
        for (int k = 0; k < per; ++k) {
            v[k] = s_d[lane * per + k];
            sum += v[k];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int run = incl - sum;
#pragma unroll
        for (int k = 0; k < per; ++k) {
            run += v[k];
            const int dd = lane * per + k;
            hist[(size_t)blockIdx.x * kRadixMax + dd] = (unsigned)run;
            if (run) {
                atomicAdd(&totals[dd], (unsigned)run);
                atomicAdd(&gtot[(blockIdx.x / kScanGroup) * kRadixMax + dd], (unsigned)run);
            }
        }
    }
}

// First stable pass of the fused binning: per tile of 2048 consecutive pairs
// of the rank-order stream, stage the ranks that own them (offsets, ids,
// packed rectangles; three independent coalesced loads), generate the pairs
// (thread t: tile slots 8t .. 8t+7, one binary search for the first slot,
// then a walk), and hand them to scatter_tile ranked by tx.
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock, 4)
k_gen_scatter(int N, const unsigned* __restrict__ order, const unsigned* __restrict__ pair_off,
              const unsigned* __restrict__ rc_rank, const unsigned char* __restrict__ sub_rank,
              const unsigned* __restrict__ n_ptr, const unsigned* __restrict__ owner_lo, int bits,
              const unsigned* __restrict__ hist, const unsigned* __restrict__ totals,
              const unsigned* __restrict__ gtot, unsigned* __restrict__ keys_out, unsigned* __restrict__ vals_out) {
    pdl_enter();
    using C = RadixCfg<MAXB>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const ScatterSmem<MAXB> sm(smem_raw, kPadTile);
    unsigned* s_off = sm.vals + kPadTile;  // [kGenWin] staged pair offsets
    unsigned* s_g = s_off + kGenWin;      // [kGenWin] staged ids
    unsigned* s_rc = s_g + kGenWin;       // [kGenWin] staged packed rectangles
    unsigned char* s_sb = reinterpret_cast<unsigned char*>(s_rc + kGenWin);  // [kGenWin] staged sub_offsets
    const int radix = 1 << bits;
    const unsigned mask = radix - 1;
    chunk_bases(hist, totals, gtot, radix, sm.base);
    const unsigned P = *n_ptr;
    unsigned lo, hi;
    chunk_of<MAXB>(P, lo, hi);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // rank data of this thread's slot in the first staging round of the
    // current tile, loaded while the previous tile was generated and scattered
    unsigned r0 = lo < hi ? owner_lo[blockIdx.x] : 0u;
    auto load_rank = [&](unsigned r, unsigned& off, unsigned& g, unsigned& rc, unsigned& sb) {
        const bool inr = r < (unsigned)N;
        off = inr ? pair_off[r] : 0xFFFFFFFFu;
        g = inr ? order[r] : 0u;
        rc = inr ? rc_rank[r] : 0u;
        sb = inr ? sub_rank[r] : 0u;
    };
    unsigned f_off, f_g, f_rc, f_sb;
    load_rank(r0 + threadIdx.x, f_off, f_g, f_rc, f_sb);
    for (unsigned base = lo; base < hi; base += C::kTileKeys) {
        const unsigned tile_n = min((unsigned)C::kTileKeys, hi - base);
        const unsigned end = base + tile_n;
        __syncthreads();  // the previous tile is finished with the staging arrays
        // stage the ranks with offsets below `end` (a prefix: offsets of
        // visible ranks increase strictly, culled ranks sit at P); every
        // loaded offset is kept, so the first rank past the tile is known too
        unsigned nr = 0;
        for (int round = 0; round * kSortBlock < kGenWin; ++round) {
            const unsigned idx = round * kSortBlock + threadIdx.x;
            unsigned off, g, rc, sb;
            if (round == 0) {
                off = f_off;
                g = f_g;
                rc = f_rc;
                sb = f_sb;
            } else {
                load_rank(r0 + idx, off, g, rc, sb);
            }
            const bool in = off < end;
            s_off[idx] = off;
            if (in) {
                s_g[idx] = g;
                s_rc[idx] = rc;
                s_sb[idx] = (unsigned char)sb;
            }
            const int c = __syncthreads_count(in);
            nr += (unsigned)c;
            if (c < kSortBlock) break;
        }
        // owner of the next tile's first pair: the next rank if it starts
        // there (its offset is staged at nr: nr < kGenWin), else the last one
        // of this tile; its first staging round is loaded now
        const unsigned nx = r0 + nr;
        const unsigned off_nx = nr < (unsigned)kGenWin ? s_off[nr] : (nx < (unsigned)N ? pair_off[nx] : 0xFFFFFFFFu);
        r0 = (nx < (unsigned)N && off_nx == end) ? nx : nx - 1;
        if (end < hi) load_rank(r0 + threadIdx.x, f_off, f_g, f_rc, f_sb);
        // generate this thread's slots into the padded key/value arrays
        const unsigned q0 = threadIdx.x * C::kItems;
        if (q0 < tile_n) {
            unsigned p = base + q0;
            unsigned i = 0, top = nr;
            while (top - i > 1) {
                const unsigned mid = (i + top) >> 1;
                if (s_off[mid] <= p) i = mid; else top = mid;
            }
            unsigned rc = s_rc[i], g = s_g[i], sb = s_sb[i];
            int x0 = rect_x0(rc), x1 = x0 + rect_w(rc);
            const unsigned w = (unsigned)(x1 - x0);
            const unsigned local = p - s_off[i];
            unsigned qq = (unsigned)__fdividef((float)local, (float)w);
            int rr = (int)local - (int)(qq * w);
            if (rr < 0) { --qq; rr += (int)w; }
            else if (rr >= (int)w) { ++qq; rr -= (int)w; }
            int tx = x0 + rr, ty = rect_y0(rc) + (int)qq;
#pragma unroll
            for (int j = 0; j < C::kItems; ++j) {
                const unsigned q = q0 + j;
                if (q < tile_n) {
                    sm.keys[pad_idx(q)] = cell_pair_key(rc, sb, tx, ty);
                    sm.vals[pad_idx(q)] = g;
                    ++p;
                    if (i + 1 < nr && s_off[i + 1] == p) {
                        ++i;
                        rc = s_rc[i];
                        g = s_g[i];
                        sb = s_sb[i];
                        x0 = rect_x0(rc);
                        x1 = x0 + rect_w(rc);
                        tx = x0;
                        ty = rect_y0(rc);
                    } else if (++tx == x1) {
                        tx = x0;
                        ++ty;
                    }
                }
            }
        }
        __syncthreads();
        unsigned key[C::kItems], val[C::kItems], d[C::kItems];
        const unsigned wq = warp * C::kWarpKeys;
#pragma unroll
        for (int j = 0; j < C::kItems; ++j) {
            const unsigned q = wq + j * 32 + lane;
            const bool valid = q < tile_n;
            key[j] = valid ? sm.keys[pad_idx(q)] : 0u;
            val[j] = valid ? sm.vals[pad_idx(q)] : 0u;
            d[j] = valid ? key[j] & mask : kNoDigit;
        }
        // scatter_tile's first barrier orders these reads before its regroup
        scatter_tile<MAXB>(sm, key, val, d, tile_n, 0, bits, keys_out, vals_out, nullptr, 0);
    }
}

template <int MAXB>
constexpr size_t gen_scatter_smem() {
    return ScatterSmem<MAXB>::bytes(kPadTile) + 3 * (size_t)kGenWin * sizeof(unsigned) + (size_t)kGenWin;
}

// Exclusive scan of one value per thread across a CTA of 1024 threads;
// returns this thread's exclusive prefix, and the total in *total.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned x, unsigned* s_w, unsigned* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    __syncthreads();  // s_w of an earlier call is consumed
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const unsigned t = s_w[lane];
        unsigned ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        s_w[lane] = ti - t;
        if (lane == 31) s_w[32] = ti;
    }
    __syncthreads();
    *total = s_w[32];
    return s_w[warp] + incl - x;
}

// A cell's range [start, end) of the cell-sorted list as the last cell pass
// left it (start > end for a cell without pairs: then (0, 0)).
__device__ __forceinline__ uint2 cell_range(const uint2* __restrict__ rg2, int c) {
    const uint2 r = rg2[c];
    return r.x < r.y ? r : make_uint2(0u, 0u);
}

// Segments of the cell lists (one CTA): cell c gets ceil(len / kSeg)
// segments, numbered in cell order; cell_seg0[c] is its first.  The ranges
// and first segments of up to kSegCache cells stay in shared memory for the
// second phase (one warp per cell, one lane per segment: coalesced writes).
constexpr int kSegCache = 2048;

__global__ void __launch_bounds__(1024)
k_seg_table(int S, const unsigned* __restrict__ cell_ranges, unsigned* __restrict__ cell_seg0,
            unsigned* __restrict__ seg_cell, unsigned* __restrict__ seg_lo, unsigned* __restrict__ seg_hi,
            SortMisc* __restrict__ misc) {
    pdl_enter();
    __shared__ unsigned s_w[33];
    __shared__ uint2 s_rg[kSegCache];
    __shared__ unsigned s_s0[kSegCache];
    const uint2* rg2 = reinterpret_cast<const uint2*>(cell_ranges);
    const int per = (S + 1023) / 1024;
    const int c0 = threadIdx.x * per;
    unsigned local = 0;
    for (int k = 0; k < per; ++k) {
        const int c = c0 + k;
        if (c < S) {
            const uint2 r = cell_range(rg2, c);
            if (c < kSegCache) s_rg[c] = r;
            local += (r.y - r.x + kSeg - 1) / kSeg;
        }
    }
    unsigned total;
    unsigned run = block_exclusive_scan(local, s_w, &total);
    for (int k = 0; k < per; ++k) {
        const int c = c0 + k;
        if (c < S) {
            const uint2 r = c < kSegCache ? s_rg[c] : cell_range(rg2, c);
            cell_seg0[c] = run;
            if (c < kSegCache) s_s0[c] = run;
            run += (r.y - r.x + kSeg - 1) / kSeg;
        }
    }
    if (threadIdx.x == 0) {
        cell_seg0[S] = total;
        misc->nseg = total;
    }
    __syncthreads();
    // one warp per cell writes the cell's segments, one lane per segment
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int c = warp; c < S; c += 32) {
        const uint2 r = c < kSegCache ? s_rg[c] : cell_range(rg2, c);
        const unsigned s0 = c < kSegCache ? s_s0[c] : cell_seg0[c];
        for (unsigned j = lane; r.x + j * kSeg < r.y; j += 32) {
            const unsigned lo = r.x + j * kSeg;
            seg_cell[s0 + j] = (unsigned)c;
            seg_lo[s0 + j] = lo;
            seg_hi[s0 + j] = min(r.y, lo + kSeg);
        }
    }
}

// Tile counts of a warp's masks, packed: bit b of a mask becomes byte b & 3
// of word b >> 2 (a 4-bit slice spread to 4 bytes by one multiply, the
// shifted copies disjoint), so one add per word counts 4 tiles and one
// warp-wide add per word sums the warp (each byte stays below 256 as long as
// no lane adds more than 7 masks).
__device__ __forceinline__ unsigned spread4(unsigned x) { return (x * 0x00204081u) & 0x01010101u; }
__device__ __forceinline__ void add_mask(unsigned (&acc)[kCellTiles / 4], unsigned m) {
#pragma unroll
    for (int j = 0; j < kCellTiles / 4; ++j) acc[j] += spread4((m >> (4 * j)) & 15u);
}
__device__ __forceinline__ unsigned packed_count(const unsigned (&acc)[kCellTiles / 4], int b) {
    return (acc[b >> 2] >> (8 * (b & 3))) & 255u;
}

// Per segment: count, per tile of its cell, the segment's Gaussians touching
// it (packed byte counters, see add_mask), from the tile masks the cell-pair
// keys carry.
__global__ void __launch_bounds__(kSortBlock)
k_seg_count(const unsigned* __restrict__ ckeys, const unsigned* __restrict__ seg_lo,
            const unsigned* __restrict__ seg_hi, const SortMisc* __restrict__ misc, unsigned* __restrict__ seg_cnt) {
    pdl_enter();
    __shared__ unsigned s_c[kSortBlock / 32][kCellTiles];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned nseg = misc->nseg;
    for (unsigned k = blockIdx.x; k < nseg; k += gridDim.x) {
        const unsigned lo = seg_lo[k], hi = seg_hi[k];
        static_assert(kSeg / kSortBlock <= 7, "packed byte counters hold at most 7 masks per lane");
        // a segment holds at most kSeg entries: this thread's kJ keys are
        // loaded together
        constexpr int kJ = kSeg / kSortBlock;
        unsigned acc[kCellTiles / 4] = {};
        unsigned key[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const unsigned i = lo + (unsigned)(j * kSortBlock) + threadIdx.x;
            key[j] = i < hi ? ckeys[i] : 0u;  // a key of 0 carries no tile
        }
#pragma unroll
        for (int j = 0; j < kJ; ++j) add_mask(acc, key_mask(key[j]));
#pragma unroll
        for (int j = 0; j < kCellTiles / 4; ++j) acc[j] = __reduce_add_sync(0xffffffffu, acc[j]);
        if (lane < kCellTiles) s_c[warp][lane] = packed_count(acc, lane);
        __syncthreads();
        if (threadIdx.x < kCellTiles) {
            unsigned t = 0;
#pragma unroll
            for (int w = 0; w < kSortBlock / 32; ++w) t += s_c[w][threadIdx.x];
            seg_cnt[(size_t)k * kCellTiles + threadIdx.x] = t;
        }
        __syncthreads();
    }
}

// One CTA per cell: exclusive prefix of the per-segment counts over the
// cell's segments, per tile bit, and the tile's total.  The cell's segments
// are cut into kCellScanGroups contiguous runs; thread (run g, tile bit b)
// sums run g's counts of bit b, the runs' sums are scanned in shared memory,
// and each thread then writes its run's bases.  All loads of a pass are
// independent, so a cell with many segments costs two rounds of latency.
constexpr int kCellScanGroups = 16;

__global__ void __launch_bounds__(kCellTiles * kCellScanGroups)
k_cell_scan(int TX, int TY, int SX, const unsigned* __restrict__ cell_seg0, const unsigned* __restrict__ seg_cnt,
            unsigned* __restrict__ seg_base, unsigned* __restrict__ tile_cnt) {
    pdl_enter();
    __shared__ unsigned s_sum[kCellScanGroups][kCellTiles];
    const unsigned c = blockIdx.x;
    const int b = threadIdx.x % kCellTiles, grp = threadIdx.x / kCellTiles;
    const unsigned k0 = cell_seg0[c], k1 = cell_seg0[c + 1];
    const unsigned n = k1 - k0;
    const unsigned per = (n + kCellScanGroups - 1) / kCellScanGroups;
    const unsigned ka = k0 + min(n, (unsigned)grp * per), kb = k0 + min(n, (unsigned)(grp + 1) * per);
    unsigned sum = 0;
    for (unsigned k = ka; k < kb; ++k) sum += seg_cnt[(size_t)k * kCellTiles + b];
    s_sum[grp][b] = sum;
    __syncthreads();
    unsigned run = 0;
    for (int g2 = 0; g2 < grp; ++g2) run += s_sum[g2][b];
    for (unsigned k = ka; k < kb; ++k) {
        const unsigned v = seg_cnt[(size_t)k * kCellTiles + b];
        seg_base[(size_t)k * kCellTiles + b] = run;
        run += v;
    }
    if (grp == kCellScanGroups - 1) {  // run is now the cell's total for bit b
        const int tx = kSuper * (int)(c % (unsigned)SX) + b % kSuper;
        const int ty = kSuper * (int)(c / (unsigned)SX) + b / kSuper;
        if (tx < TX && ty < TY) tile_cnt[ty * TX + tx] = run;
    }
}

// Exclusive scan of the tile counts in tile order (one CTA, 4096 tiles per
// round, four consecutive tiles per thread): tile starts and ranges; empty
// tiles get (0, 0).  Each round's results are gathered in shared memory
// (padded: one spare word per 32) and written out with consecutive threads
// on consecutive tiles.
constexpr int kTileRound = 4096;

__device__ __forceinline__ int pad32(int i) { return i + (i >> 5); }

__global__ void __launch_bounds__(1024)
k_tile_scan(int T, const unsigned* __restrict__ tile_cnt, unsigned* __restrict__ tile_start,
            unsigned* __restrict__ ranges) {
    pdl_enter();
    __shared__ unsigned s_w[33];
    __shared__ unsigned s_start[kTileRound + kTileRound / 32];
    __shared__ unsigned s_cnt[kTileRound + kTileRound / 32];
    uint2* rg2 = reinterpret_cast<uint2*>(ranges);
    unsigned carry = 0;
    for (int t0 = 0; t0 < T; t0 += kTileRound) {
        const int t = t0 + 4 * threadIdx.x;
        unsigned v[4], local = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[j] = t + j < T ? tile_cnt[t + j] : 0u;
            local += v[j];
        }
        unsigned total;
        unsigned run = carry + block_exclusive_scan(local, s_w, &total);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s_start[pad32(4 * threadIdx.x + j)] = run;
            s_cnt[pad32(4 * threadIdx.x + j)] = v[j];
            run += v[j];
        }
        __syncthreads();
        const int nr = min(kTileRound, T - t0);
        for (int i = threadIdx.x; i < nr; i += 1024) {
            const unsigned st = s_start[pad32(i)], n = s_cnt[pad32(i)];
            tile_start[t0 + i] = st;
            rg2[t0 + i] = n ? make_uint2(st, st + n) : make_uint2(0u, 0u);
        }
        carry += total;
        __syncthreads();  // s_start / s_cnt are rewritten next round
    }
}

// Per segment: write its Gaussians into the lists of its cell's tiles.  Per
// chunk of 256 list entries: each warp counts its Gaussians per tile bit
// (packed byte counters), one thread per bit turns the warps' counts into bases (warp
// order after the running base), then each warp writes, per tile bit, its
// Gaussians at base + ballot rank: consecutive lanes, consecutive addresses.
// Optional 64-bit (tile << 32 | depth bits) keys.
template <bool kKeys>
__global__ void __launch_bounds__(kSortBlock)
k_seg_emit(int TX, int TY, int SX, const unsigned* __restrict__ clist, const unsigned* __restrict__ ckeys,
           const float* __restrict__ depth, const unsigned* __restrict__ seg_cell,
           const unsigned* __restrict__ seg_lo, const unsigned* __restrict__ seg_hi,
           const unsigned* __restrict__ seg_base, const unsigned* __restrict__ tile_start,
           const SortMisc* __restrict__ misc, unsigned* __restrict__ ids, unsigned long long* __restrict__ keys) {
    pdl_enter();
    constexpr int kW = kSortBlock / 32;
    __shared__ unsigned s_base[kCellTiles];
    __shared__ __align__(16) unsigned s_wb[kW][kCellTiles];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
    const unsigned nseg = misc->nseg;
    for (unsigned k = blockIdx.x; k < nseg; k += gridDim.x) {
        const unsigned c = seg_cell[k], lo = seg_lo[k], hi = seg_hi[k];
        const int cx = (int)(c % (unsigned)SX), cy = (int)(c / (unsigned)SX);
        if (threadIdx.x < kCellTiles) {
            const int b = threadIdx.x;
            const int tx = kSuper * cx + b % kSuper, ty = kSuper * cy + b / kSuper;
            s_base[b] = (tx < TX && ty < TY) ? tile_start[ty * TX + tx] + seg_base[(size_t)k * kCellTiles + b] : 0u;
        }
        // a segment holds at most kSeg entries: this thread's entries and
        // masks for the whole segment are loaded together, up front
        constexpr int kJ = kSeg / kSortBlock;
        unsigned gs[kJ], ms[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const unsigned i = lo + (unsigned)(j * kSortBlock) + threadIdx.x;
            gs[j] = i < hi ? clist[i] : 0u;
            ms[j] = i < hi ? key_mask(ckeys[i]) : 0u;
        }
#pragma unroll
        for (int jc = 0; jc < kJ; ++jc) {
            const unsigned base = lo + (unsigned)(jc * kSortBlock);
            if (base >= hi) break;  // block-uniform
            const unsigned g = gs[jc];
            const unsigned m = ms[jc];
            // this warp's count per tile bit (packed byte counters)
            unsigned acc[kCellTiles / 4] = {};
            add_mask(acc, m);
#pragma unroll
            for (int j = 0; j < kCellTiles / 4; ++j) acc[j] = __reduce_add_sync(0xffffffffu, acc[j]);
            if (lane < kCellTiles) s_wb[warp][lane] = packed_count(acc, lane);
            __syncthreads();
            if (threadIdx.x < kCellTiles) {
                const int b = threadIdx.x;
                unsigned run = s_base[b];
#pragma unroll
                for (int w = 0; w < kW; ++w) {
                    const unsigned cnt = s_wb[w][b];
                    s_wb[w][b] = run;
                    run += cnt;
                }
                s_base[b] = run;
            }
            __syncthreads();
            const float dg = (kKeys && m && id_ok(g)) ? depth[g] : 0.0f;
            // tile bits in order, unrolled: no find-first-set / bit-reverse
            // (XU) instructions, and no test of the warp's union of masks
            // (a row of 32 list entries almost always touches all 16 tiles);
            // the warp's bases come four at a time
#pragma unroll
            for (int q = 0; q < kCellTiles / 4; ++q) {
                const uint4 b4 = *reinterpret_cast<const uint4*>(&s_wb[warp][4 * q]);
                const unsigned wb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int b = 4 * q + i;
                    const bool mine = (m >> b) & 1u;
                    const unsigned bal = __ballot_sync(0xffffffffu, mine);
                    if (mine) {
                        const unsigned pos = wb[i] + __popc(bal & lt);
                        if (pos_ok(pos)) {
                            ids[pos] = g;
                            if (kKeys) {
                                const unsigned t =
                                    (unsigned)((kSuper * cy + b / kSuper) * TX + kSuper * cx + b % kSuper);
                                keys[pos] = ((unsigned long long)t << 32) | __float_as_uint(dg);
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();  // s_base and s_wb are rebuilt for the next segment
    }
}

int ceil_log2(unsigned x) {
    int b = 0;
    while ((1ull << b) < x) ++b;
    return b;
}

template <int MAXB>
void enable_scatter_smem() {
    opt_in_smem(k_radix_scatter<MAXB>, RadixCfg<MAXB>::kScatterSmem);
}

template <int MAXB>
void radix_pass(cudaStream_t st, int G, const unsigned* n_ptr, int shift, int bits, const unsigned* ki,
                const unsigned* vi, unsigned* ko, unsigned* vo, unsigned* hist, unsigned* totals, unsigned* gtot,
                unsigned* cell_ranges = nullptr, int SX = 0) {
    enable_scatter_smem<MAXB>();
    launch_pdl(k_radix_hist<MAXB>, G, kSortBlock, 0, st, ki, n_ptr, shift, bits, hist, totals, gtot); note_launch();
    launch_pdl(k_radix_scatter<MAXB>, G, kSortBlock, RadixCfg<MAXB>::kScatterSmem, st, ki, vi, ko, vo, n_ptr, shift, bits,
               hist, totals, gtot, cell_ranges, SX);
    note_launch();
}

// One stable LSD radix sort of (keys, vals) over bits [0, total_bits), with
// at most 8 bits per pass.  The final pass writes to (final_keys, final_vals)
// when they are given.  Returns the number of passes.
int radix_sort(cudaStream_t st, int G, const unsigned* n_ptr, int total_bits, unsigned* k0, unsigned* v0,
               unsigned* k1, unsigned* v1, unsigned* final_vals, unsigned** out_keys, unsigned* hist,
               unsigned* totals, unsigned* gtot, int pass_base) {
    const int passes = (total_bits + 7) / 8;
    if (passes == 0) {
        *out_keys = k0;
        return 0;
    }
    const int bits = (total_bits + passes - 1) / passes;
    unsigned *ki = k0, *vi = v0, *ko = k1, *vo = v1;
    for (int p = 0; p < passes; ++p) {
        const bool last = p == passes - 1;
        unsigned* vdst = (last && final_vals) ? final_vals : vo;
        unsigned* h = hist + (size_t)(pass_base + p) * kRadixMax * kSortMaxGrid;
        unsigned* tot = totals + (size_t)(pass_base + p) * kRadixMax;
        unsigned* gt = gtot + (size_t)(pass_base + p) * kMaxGroups * kRadixMax;
        if (bits <= 7)
            radix_pass<7>(st, G, n_ptr, p * bits, bits, ki, vi, ko, vdst, h, tot, gt);
        else
            radix_pass<8>(st, G, n_ptr, p * bits, bits, ki, vi, ko, vdst, h, tot, gt);
        unsigned* tk = ki;
        ki = ko;
        ko = tk;
        unsigned* tv = vi;
        vi = vdst;
        vo = tv;
    }
    *out_keys = ki;
    return passes;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_bin_sort_ws_bytes(int N, unsigned capacity, int width, int height) {
    if (N < 0 || width < 1 || height < 1) return 0;
    return carve(nullptr, N, capacity, (width + kTile - 1) / kTile, (height + kTile - 1) / kTile, nullptr);
}

extern "C" int gs_bin_sort(const gs_camera* cam, int N, const float* depth, const int* rect,
                           const unsigned* tiles_touched, const unsigned* d_num_pairs, unsigned capacity,
                           unsigned* ids, unsigned* ranges, unsigned long long* keys, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!camera_ok(cam) || N < 0 || !d_num_pairs || !ranges || !ws) return GS_ERR_INVALID_ARG;
    if (N > 0 && (!depth || !rect || !tiles_touched)) return GS_ERR_INVALID_ARG;
    if (capacity > 0 && !ids) return GS_ERR_INVALID_ARG;
    if (!aligned(ws, 256) || ws_bytes < gs_bin_sort_ws_bytes(N, capacity, cam->width, cam->height))
        return GS_ERR_INVALID_ARG;
    if (rect && !aligned(rect, 16)) return GS_ERR_INVALID_ARG;
    if (ranges && !aligned(ranges, 8)) return GS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const int TX = tiles_x(*cam), TY = tiles_y(*cam), T = TX * TY;
    BinWs w;
    carve(ws, N, capacity, TX, TY, &w);
    const bool sup = w.n_cells > 0 && capacity > 0;  // super-tile route
    const int SX = (TX + kSuper - 1) / kSuper, SY = (TY + kSuper - 1) / kSuper;
    const int4* rect4 = reinterpret_cast<const int4*>(rect);

    {
        int work = N > 2 * T ? N : 2 * T;
        int blocks = (work + 255) / 256;
        if (blocks < 1) blocks = 1;
        if (blocks > 148 * 8) blocks = 148 * 8;
        launch_pdl(k_bin_init, blocks, 256, 0, st, N, T, depth, tiles_touched, d_num_pairs, capacity, w, ranges); note_launch();
        GS_LAUNCH_CHECK();
    }
    if (N == 0) return GS_OK;

    // 1. depth ranks of the Gaussians (32-bit keys, culled ones last)
    const int Gd = (N + 2047) / 2048 < kSortMaxGrid ? (N + 2047) / 2048 : kSortMaxGrid;
    unsigned* dkeys_sorted = nullptr;
    const int dpasses = radix_sort(st, Gd, &w.misc->n_gauss, 32, w.dkeys0, w.dvals0, w.dkeys1, w.dvals1, nullptr,
                                   &dkeys_sorted, w.hist, w.totals, w.gtot, 0);
    const unsigned* order = (dpasses % 2 == 0) ? w.dvals0 : w.dvals1;
    GS_LAUNCH_CHECK();

    // 2. pair offsets in rank order (of super-tile pairs on the super-tile route)
    const int nb = (N + kScanTile - 1) / kScanTile;
    const int Gp = (int)((capacity + 2047u) / 2048u) < kSortMaxGrid ? (int)((capacity + 2047u) / 2048u) : kSortMaxGrid;
    launch_pdl(k_scan_partials, nb, kSortBlock, 0, st, N, order, tiles_touched, sup ? rect4 : nullptr, w.cnt_rank,
                                               w.rc_rank, w.sub_rank, w.scan_part, w.misc); note_launch();
    launch_pdl(k_scan_down, nb, kSortBlock, 0, st, N, w.cnt_rank, w.scan_part, w.pair_off, w.misc,
                                           (unsigned)(Gp < 1 ? 1 : Gp), sup ? w.owner_lo : nullptr, w.owner_hi); note_launch();
    GS_LAUNCH_CHECK();
    if (capacity == 0) return GS_OK;

    if (sup) {
        // 3'. super-tile route: bin to cells (generate + stable pass on cx,
        //     stable pass on cy), cell ranges, segments, per-tile counts,
        //     tile ranges, expansion into the tile lists
        const unsigned* ps = &w.misc->ps;
        const int bx = ceil_log2((unsigned)SX), by = ceil_log2((unsigned)SY);
        unsigned* h1 = w.hist + (size_t)4 * kRadixMax * kSortMaxGrid;
        unsigned* t1 = w.totals + (size_t)4 * kRadixMax;
        unsigned* g1 = w.gtot + (size_t)4 * kMaxGroups * kRadixMax;
        if (bx <= 7) {
            launch_pdl(k_gen_hist<7>, Gp, kSortBlock, 0, st, w.pair_off, w.rc_rank, ps, w.owner_lo, w.owner_hi, h1, t1,
                       g1);
            note_launch();
            opt_in_smem(k_gen_scatter<7>, gen_scatter_smem<7>());
            launch_pdl(k_gen_scatter<7>, Gp, kSortBlock, gen_scatter_smem<7>(), st, N, order, w.pair_off, w.rc_rank,
                       w.sub_rank, ps, w.owner_lo, bx, h1, t1, g1, w.tkeys0, w.tvals0);
            note_launch();
        } else {
            launch_pdl(k_gen_hist<8>, Gp, kSortBlock, 0, st, w.pair_off, w.rc_rank, ps, w.owner_lo, w.owner_hi, h1, t1,
                       g1);
            note_launch();
            opt_in_smem(k_gen_scatter<8>, gen_scatter_smem<8>());
            launch_pdl(k_gen_scatter<8>, Gp, kSortBlock, gen_scatter_smem<8>(), st, N, order, w.pair_off, w.rc_rank,
                       w.sub_rank, ps, w.owner_lo, bx, h1, t1, g1, w.tkeys0, w.tvals0);
            note_launch();
        }
        GS_LAUNCH_CHECK();
        unsigned* h2 = w.hist + (size_t)5 * kRadixMax * kSortMaxGrid;
        unsigned* t2 = w.totals + (size_t)5 * kRadixMax;
        unsigned* g2 = w.gtot + (size_t)5 * kMaxGroups * kRadixMax;
        // the cy pass also records each cell's range of the sorted list
        if (by <= 7)
            radix_pass<7>(st, Gp, ps, 16, by, w.tkeys0, w.tvals0, w.tkeys1, w.tvals1, h2, t2, g2, w.cell_ranges, SX);
        else
            radix_pass<8>(st, Gp, ps, 16, by, w.tkeys0, w.tvals0, w.tkeys1, w.tvals1, h2, t2, g2, w.cell_ranges, SX);
        GS_LAUNCH_CHECK();
        const int S = SX * SY;
        launch_pdl(k_seg_table, 1, 1024, 0, st, S, w.cell_ranges, w.cell_seg0, w.seg_cell, w.seg_lo, w.seg_hi, w.misc); note_launch();
        const int gseg = (int)(w.max_seg < 148u * 8u ? w.max_seg : 148u * 8u);
        launch_pdl(k_seg_count, gseg, kSortBlock, 0, st, w.tkeys1, w.seg_lo, w.seg_hi, w.misc, w.seg_cnt); note_launch();
        launch_pdl(k_cell_scan, S, kCellTiles * kCellScanGroups, 0, st, TX, TY, SX, w.cell_seg0, w.seg_cnt, w.seg_base, w.tile_cnt); note_launch();
        launch_pdl(k_tile_scan, 1, 1024, 0, st, T, w.tile_cnt, w.tile_start, ranges); note_launch();
        if (keys)
            launch_pdl(k_seg_emit<true>, gseg, kSortBlock, 0, st, TX, TY, SX, w.tvals1, w.tkeys1, depth, w.seg_cell,
                       w.seg_lo, w.seg_hi, w.seg_base, w.tile_start, w.misc, ids, keys);
        else
            launch_pdl(k_seg_emit<false>, gseg, kSortBlock, 0, st, TX, TY, SX, w.tvals1, w.tkeys1, depth, w.seg_cell,
                       w.seg_lo, w.seg_hi, w.seg_base, w.tile_start, w.misc, ids, keys);
        note_launch();
        GS_LAUNCH_CHECK();
        return GS_OK;
    }

    // 3. emit pairs in rank order, then a stable sort by tile id
    const int tile_bits = ceil_log2((unsigned)T);
    const int tpasses = (tile_bits + 7) / 8;
    {
        // one CTA per 2048 output pairs, up to a few waves (grid-stride beyond)
        unsigned segs = (capacity + kEmitSeg - 1) / kEmitSeg;
        int blocks = segs > 148u * 32u ? 148 * 32 : (int)segs;
        if (blocks < 1) blocks = 1;
        unsigned* emit_vals = tpasses == 0 ? ids : w.tvals0;
        launch_pdl(k_emit, blocks, kSortBlock, 0, st, N, TX, order, w.pair_off, reinterpret_cast<const int4*>(rect),
                                              tiles_touched, w.misc, w.tkeys0, emit_vals); note_launch();
        GS_LAUNCH_CHECK();
    }
    unsigned* tkeys_sorted = nullptr;
    radix_sort(st, Gp, &w.misc->p_eff, tile_bits, w.tkeys0, w.tvals0, w.tkeys1, w.tvals1, ids, &tkeys_sorted,
               w.hist, w.totals, w.gtot, 4);
    GS_LAUNCH_CHECK();

    // 4. tile ranges (and optional 64-bit keys)
    {
        int blocks = (int)((capacity + 1023u) / 1024u);
        if (blocks > 148 * 16) blocks = 148 * 16;
        if (blocks < 1) blocks = 1;
        launch_pdl(k_ranges, blocks, 256, 0, st, tkeys_sorted, ids, depth, w.misc, ranges, keys); note_launch();
        GS_LAUNCH_CHECK();
    }
    return GS_OK;
}