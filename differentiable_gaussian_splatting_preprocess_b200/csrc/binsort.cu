// Tile binning and (tile, depth) ordering.
//
// "4-3DGS训练与优化" section E.3: each projected Gaussian's AABB selects the
// tiles it may touch; the Gaussians of each tile are sorted by depth and
// splatted in that order; tiles are independent.  "Gaussian Splatting反向传播的
// CUDA实现" section 1: the sorted list and the per-tile ranges are kept and
// reused by the backward.
//
// The order produced is that of a sort of 64-bit keys (tile << 32 |
// float_bits(depth)) with ties broken by Gaussian id.  It is reached in two
// sorts instead of one wide one:
//   1. the N Gaussians are sorted by depth bits (stable LSD radix sort, 8-bit
//      digits, ids in increasing order initially, culled ones last), which
//      gives every visible Gaussian its (depth, id) rank;
//   2. the (tile, Gaussian) pairs are emitted in rank order and stably sorted
//      by tile id alone (ceil(log2 T) bits, at most 8 per pass).
// A stable sort by tile of a list already in (depth, id) order yields the
// (tile, depth, id) order, so the result is the same as the 64-bit sort while
// the pair-sized passes only move the tile bits.
//
// Every kernel is a plain grid over its data; there are no inter-block waits.

#include <cuda_runtime.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kSortBlock = 256;
constexpr int kSortMaxGrid = 148 * 4;  // CTAs per radix pass: a multiple of the SM count
constexpr int kRadixMax = 256;
constexpr int kMaxPasses = 8;          // 4 depth passes + up to 3 tile passes (+1 spare)
constexpr int kScanItems = 8;          // items per thread in the rank-order scan
constexpr int kScanTile = kSortBlock * kScanItems;

struct SortMisc {
    unsigned n_gauss;    // N
    unsigned p_eff;      // P if it fits the capacity, else 0
    unsigned pad[62];
};

struct BinWs {
    WsHeader* hdr;
    SortMisc* misc;
    unsigned *dkeys0, *dvals0, *dkeys1, *dvals1;  // depth sort, N each
    unsigned* pair_off;                            // N + 1
    unsigned* scan_part;                           // ceil(N / kScanTile) + 1
    unsigned *tkeys0, *tvals0, *tkeys1, *tvals1;   // pair sort, capacity each
    unsigned* hist;                                // kMaxPasses * kRadixMax * kSortMaxGrid
    unsigned* totals;                              // kMaxPasses * kRadixMax
};

size_t carve(void* base, int N, unsigned capacity, BinWs* w) {
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
    t.scan_part = (unsigned*)take(((n + kScanTile - 1) / kScanTile + 1) * 4);
    t.tkeys0 = (unsigned*)take(cap * 4);
    t.tvals0 = (unsigned*)take(cap * 4);
    t.tkeys1 = (unsigned*)take(cap * 4);
    t.tvals1 = (unsigned*)take(cap * 4);
    t.hist = (unsigned*)take((size_t)kMaxPasses * kRadixMax * kSortMaxGrid * 4);
    t.totals = (unsigned*)take((size_t)kMaxPasses * kRadixMax * 4);
    if (w) *w = t;
    return off;
}

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
    const int stride = gridDim.x * blockDim.x;
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = tid; i < 2 * T; i += stride) ranges[i] = 0u;
    for (int i = tid; i < kMaxPasses * kRadixMax; i += stride) w.totals[i] = 0u;
    for (int i = tid; i < N; i += stride) {
        w.dkeys0[i] = tiles_touched[i] > 0 ? __float_as_uint(depth[i]) : 0xFFFFFFFFu;
        w.dvals0[i] = (unsigned)i;
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

template <int MAXB>
__device__ __forceinline__ void chunk_of(unsigned n, unsigned& lo, unsigned& hi) {
    constexpr unsigned tile = RadixCfg<MAXB>::kTileKeys;
    const unsigned G = gridDim.x;
    unsigned chunk = (n + G - 1) / G;
    chunk = (chunk + tile - 1) / tile * tile;
    const unsigned long long l = (unsigned long long)blockIdx.x * chunk;
    lo = l < n ? (unsigned)l : n;
    hi = min(n, lo + chunk);
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

// Per-CTA digit histogram of its chunk, stored digit-major (hist[d * G + cta]);
// digit totals accumulate into totals[d].  Each warp counts into its own
// shared-memory histogram.
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock)
k_radix_hist(const unsigned* __restrict__ keys, const unsigned* __restrict__ n_ptr, int shift, int bits,
             unsigned* __restrict__ hist, unsigned* __restrict__ totals) {
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
    const unsigned G = gridDim.x;
    for (int dd = threadIdx.x; dd < radix; dd += kSortBlock) {
        unsigned c = 0;
#pragma unroll
        for (int w = 0; w < C::kWarps; ++w) c += s_h[w][dd];
        hist[(size_t)dd * G + blockIdx.x] = c;
        if (c) atomicAdd(&totals[dd], c);
    }
}

// One CTA per digit d: offsets[d][c] = (sum of totals below d) + exclusive
// prefix over CTAs of hist[d][.], in place.
__global__ void __launch_bounds__(kSortBlock)
k_radix_scan(unsigned* __restrict__ hist, const unsigned* __restrict__ totals, int G) {
    const int d = blockIdx.x;
    __shared__ unsigned s_w[kSortBlock / 32];
    __shared__ unsigned s_base;
    unsigned b = 0;
    for (int e = threadIdx.x; e < d; e += kSortBlock) b += totals[e];
    b = __reduce_add_sync(0xffffffffu, b);
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned s2 = 0;
        for (int k = 0; k < kSortBlock / 32; ++k) s2 += s_w[k];
        s_base = s2;
    }
    __syncthreads();
    const int per = (G + kSortBlock - 1) / kSortBlock;
    unsigned* row = hist + (size_t)d * G;
    const int c0 = threadIdx.x * per;
    unsigned local = 0;
    for (int k = 0; k < per; ++k)
        if (c0 + k < G) local += row[c0 + k];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    __syncthreads();
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    unsigned wbase = 0;
    for (int k = 0; k < warp; ++k) wbase += s_w[k];
    unsigned run = s_base + wbase + incl - local;
    for (int k = 0; k < per; ++k)
        if (c0 + k < G) {
            const unsigned c = row[c0 + k];
            row[c0 + k] = run;
            run += c;
        }
}

// Stable scatter.  Per tile of 2048 keys, each warp owning a contiguous block
// of 256 of them (8 rows of 32):
//   1. each warp ranks its keys row by row (digit_peers within the row, plus
//      a running per-digit count of the warp's earlier rows), so ranks follow
//      input order within the warp;
//   2. one thread per digit turns the warps' counts into offsets (warp
//      order), giving the tile's count per digit; one warp scans those into
//      tile-local digit starts and advances the running global bases;
//   3. every key is placed in shared memory at its tile-local sorted position;
//   4. the regrouped tile is written out in order, so consecutive lanes write
//      consecutive addresses of one digit's run (coalesced stores).
template <int MAXB>
__global__ void __launch_bounds__(kSortBlock)
k_radix_scatter(const unsigned* __restrict__ keys_in, const unsigned* __restrict__ vals_in,
                unsigned* __restrict__ keys_out, unsigned* __restrict__ vals_out,
                const unsigned* __restrict__ n_ptr, int shift, int bits, const unsigned* __restrict__ offsets) {
    using C = RadixCfg<MAXB>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned* s_base = reinterpret_cast<unsigned*>(smem_raw);   // [radix] running global base
    unsigned* s_tcnt = s_base + C::kRadix;                      // [radix] this tile's count per digit
    unsigned* s_tstart = s_tcnt + C::kRadix;                    // [radix] tile-local start per digit
    unsigned* s_tbase = s_tstart + C::kRadix;                   // [radix] global base for this tile
    unsigned* s_wcnt = s_tbase + C::kRadix;                     // [warps][radix] counts, then offsets
    unsigned* s_keys = s_wcnt + C::kWarps * C::kRadix;          // [tile] regrouped keys
    unsigned* s_vals = s_keys + C::kTileKeys;                   // [tile] regrouped values
    const int radix = 1 << bits;
    const unsigned mask = radix - 1;
    const unsigned G = gridDim.x;
    for (int dd = threadIdx.x; dd < radix; dd += kSortBlock) s_base[dd] = offsets[(size_t)dd * G + blockIdx.x];
    unsigned lo, hi;
    chunk_of<MAXB>(*n_ptr, lo, hi);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = lanemask_lt();
    unsigned* wcnt = s_wcnt + warp * C::kRadix;
    for (unsigned base = lo; base < hi; base += C::kTileKeys) {
        const unsigned tile_n = min((unsigned)C::kTileKeys, hi - base);
        for (int dd = lane; dd < radix; dd += 32) wcnt[dd] = 0;
        __syncwarp();
        unsigned key[C::kItems], val[C::kItems], d[C::kItems], rank[C::kItems];
        const unsigned wbase = base + warp * C::kWarpKeys;
#pragma unroll
        for (int j = 0; j < C::kItems; ++j) {
            const unsigned i = wbase + j * 32 + lane;
            const bool valid = i < hi;
            key[j] = valid ? keys_in[i] : 0u;
            val[j] = valid ? vals_in[i] : 0u;
            d[j] = valid ? (key[j] >> shift) & mask : kNoDigit;
        }
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
                const unsigned c = s_wcnt[w * C::kRadix + dd];
                s_wcnt[w * C::kRadix + dd] = run;
                run += c;
            }
            s_tcnt[dd] = run;
        }
        __syncthreads();
        if (warp == 0) {
            constexpr int per = (C::kRadix + 31) / 32;
            unsigned v[per], sum = 0;
#pragma unroll
            for (int k = 0; k < per; ++k) {
                const int dd = lane * per + k;
                v[k] = dd < radix ? s_tcnt[dd] : 0u;
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
                    s_tstart[dd] = run;
                    s_tbase[dd] = s_base[dd];
                    s_base[dd] += v[k];
                }
                run += v[k];
            }
        }
        __syncthreads();
        // 3. regroup the tile by digit in shared memory
#pragma unroll
        for (int j = 0; j < C::kItems; ++j) {
            if (d[j] != kNoDigit) {
                const unsigned loc = s_tstart[d[j]] + wcnt[d[j]] + rank[j];
                s_keys[loc] = key[j];
                s_vals[loc] = val[j];
            }
        }
        __syncthreads();
        // 4. write the regrouped tile: consecutive q of one digit go to
        //    consecutive output positions
        for (unsigned q = threadIdx.x; q < tile_n; q += kSortBlock) {
            const unsigned k2 = s_keys[q];
            const unsigned dq = (k2 >> shift) & mask;
            const unsigned pos = s_tbase[dq] + (q - s_tstart[dq]);
            keys_out[pos] = k2;
            vals_out[pos] = s_vals[q];
        }
        __syncthreads();  // the next tile reuses every shared array
    }
}

// Exclusive scan, in depth-rank order, of the pair counts:
// pair_off[r] = sum over ranks r' < r of tiles_touched[order[r']].
__global__ void __launch_bounds__(kSortBlock)
k_scan_partials(int N, const unsigned* __restrict__ order, const unsigned* __restrict__ tiles_touched,
                unsigned* __restrict__ part) {
    const int base = blockIdx.x * kScanTile;
    unsigned s = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k * kSortBlock + threadIdx.x;
        if (r < N) s += tiles_touched[order[r]];
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

__global__ void __launch_bounds__(1024) k_scan_top(unsigned* __restrict__ part, int nb) {
    // exclusive scan of nb partial sums by one CTA, each thread a contiguous run
    __shared__ unsigned s_w[32];
    const int per = (nb + 1023) / 1024;
    const int c0 = threadIdx.x * per;
    unsigned local = 0;
    for (int k = 0; k < per; ++k)
        if (c0 + k < nb) local += part[c0 + k];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    unsigned wbase = 0;
    for (int k = 0; k < warp; ++k) wbase += s_w[k];
    unsigned run = wbase + incl - local;
    for (int k = 0; k < per; ++k)
        if (c0 + k < nb) {
            const unsigned c = part[c0 + k];
            part[c0 + k] = run;
            run += c;
        }
}

__global__ void __launch_bounds__(kSortBlock)
k_scan_down(int N, const unsigned* __restrict__ order, const unsigned* __restrict__ tiles_touched,
            const unsigned* __restrict__ part, unsigned* __restrict__ pair_off) {
    // each thread owns kScanItems consecutive ranks
    const int base = blockIdx.x * kScanTile + threadIdx.x * kScanItems;
    unsigned v[kScanItems];
    unsigned local = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k;
        v[k] = r < N ? tiles_touched[order[r]] : 0u;
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
    __syncthreads();
    unsigned wbase = 0;
    for (int k = 0; k < warp; ++k) wbase += s_w[k];
    unsigned run = part[blockIdx.x] + wbase + incl - local;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        const int r = base + k;
        if (r < N) pair_off[r] = run;
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
       const int4* __restrict__ rect, const unsigned* __restrict__ tiles_touched, const SortMisc* __restrict__ misc,
       unsigned* __restrict__ tkeys, unsigned* __restrict__ tvals) {
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
                if (keys) keys[k] = ((unsigned long long)t[j] << 32) | __float_as_uint(depth[ids[k]]);
            }
        }
    }
}

int ceil_log2(unsigned x) {
    int b = 0;
    while ((1ull << b) < x) ++b;
    return b;
}

// The scatter needs more than the default 48 KiB of dynamic shared memory;
// the attribute belongs to the current device, so it is set before each use.
template <int MAXB>
void enable_scatter_smem() {
    cudaFuncSetAttribute(k_radix_scatter<MAXB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)RadixCfg<MAXB>::kScatterSmem);
}

template <int MAXB>
void radix_pass(cudaStream_t st, int G, const unsigned* n_ptr, int shift, int bits, const unsigned* ki,
                const unsigned* vi, unsigned* ko, unsigned* vo, unsigned* hist, unsigned* totals) {
    enable_scatter_smem<MAXB>();
    k_radix_hist<MAXB><<<G, kSortBlock, 0, st>>>(ki, n_ptr, shift, bits, hist, totals);
    k_radix_scan<<<1 << bits, kSortBlock, 0, st>>>(hist, totals, G);
    k_radix_scatter<MAXB><<<G, kSortBlock, RadixCfg<MAXB>::kScatterSmem, st>>>(ki, vi, ko, vo, n_ptr, shift, bits,
                                                                                hist);
}

// One stable LSD radix sort of (keys, vals) over bits [0, total_bits), with
// at most 8 bits per pass.  The final pass writes to (final_keys, final_vals)
// when they are given.  Returns the number of passes.
int radix_sort(cudaStream_t st, int G, const unsigned* n_ptr, int total_bits, unsigned* k0, unsigned* v0,
               unsigned* k1, unsigned* v1, unsigned* final_vals, unsigned** out_keys, unsigned* hist,
               unsigned* totals, int pass_base) {
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
        if (bits <= 7)
            radix_pass<7>(st, G, n_ptr, p * bits, bits, ki, vi, ko, vdst, h, tot);
        else
            radix_pass<8>(st, G, n_ptr, p * bits, bits, ki, vi, ko, vdst, h, tot);
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

extern "C" size_t gs_bin_sort_ws_bytes(int N, unsigned capacity) {
    if (N < 0) return 0;
    return carve(nullptr, N, capacity, nullptr);
}

extern "C" int gs_bin_sort(const gs_camera* cam, int N, const float* depth, const int* rect,
                           const unsigned* tiles_touched, const unsigned* d_num_pairs, unsigned capacity,
                           unsigned* ids, unsigned* ranges, unsigned long long* keys, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!camera_ok(cam) || N < 0 || !d_num_pairs || !ranges || !ws) return GS_ERR_INVALID_ARG;
    if (N > 0 && (!depth || !rect || !tiles_touched)) return GS_ERR_INVALID_ARG;
    if (capacity > 0 && !ids) return GS_ERR_INVALID_ARG;
    if (!aligned(ws, 256) || ws_bytes < gs_bin_sort_ws_bytes(N, capacity)) return GS_ERR_INVALID_ARG;
    if (rect && !aligned(rect, 16)) return GS_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    BinWs w;
    carve(ws, N, capacity, &w);
    const int TX = tiles_x(*cam), TY = tiles_y(*cam), T = TX * TY;

    {
        int work = N > 2 * T ? N : 2 * T;
        int blocks = (work + 255) / 256;
        if (blocks < 1) blocks = 1;
        if (blocks > 148 * 8) blocks = 148 * 8;
        k_bin_init<<<blocks, 256, 0, st>>>(N, T, depth, tiles_touched, d_num_pairs, capacity, w, ranges);
        GS_LAUNCH_CHECK();
    }
    if (N == 0) return GS_OK;

    // 1. depth ranks of the Gaussians (32-bit keys, culled ones last)
    const int Gd = (N + 2047) / 2048 < kSortMaxGrid ? (N + 2047) / 2048 : kSortMaxGrid;
    unsigned* dkeys_sorted = nullptr;
    const int dpasses = radix_sort(st, Gd, &w.misc->n_gauss, 32, w.dkeys0, w.dvals0, w.dkeys1, w.dvals1, nullptr,
                                   &dkeys_sorted, w.hist, w.totals, 0);
    const unsigned* order = (dpasses % 2 == 0) ? w.dvals0 : w.dvals1;
    GS_LAUNCH_CHECK();

    // 2. pair offsets in rank order
    const int nb = (N + kScanTile - 1) / kScanTile;
    k_scan_partials<<<nb, kSortBlock, 0, st>>>(N, order, tiles_touched, w.scan_part);
    k_scan_top<<<1, 1024, 0, st>>>(w.scan_part, nb);
    k_scan_down<<<nb, kSortBlock, 0, st>>>(N, order, tiles_touched, w.scan_part, w.pair_off);
    GS_LAUNCH_CHECK();
    if (capacity == 0) return GS_OK;

    // 3. emit pairs in rank order, then a stable sort by tile id
    const int tile_bits = ceil_log2((unsigned)T);
    const int tpasses = (tile_bits + 7) / 8;
    {
        // one CTA per 2048 output pairs, up to a few waves (grid-stride beyond)
        unsigned segs = (capacity + kEmitSeg - 1) / kEmitSeg;
        int blocks = segs > 148u * 32u ? 148 * 32 : (int)segs;
        if (blocks < 1) blocks = 1;
        unsigned* emit_vals = tpasses == 0 ? ids : w.tvals0;
        k_emit<<<blocks, kSortBlock, 0, st>>>(N, TX, order, w.pair_off, reinterpret_cast<const int4*>(rect),
                                              tiles_touched, w.misc, w.tkeys0, emit_vals);
        GS_LAUNCH_CHECK();
    }
    const int Gp = (int)((capacity + 2047u) / 2048u) < kSortMaxGrid ? (int)((capacity + 2047u) / 2048u) : kSortMaxGrid;
    unsigned* tkeys_sorted = nullptr;
    radix_sort(st, Gp, &w.misc->p_eff, tile_bits, w.tkeys0, w.tvals0, w.tkeys1, w.tvals1, ids, &tkeys_sorted,
               w.hist, w.totals, 4);
    GS_LAUNCH_CHECK();

    // 4. tile ranges (and optional 64-bit keys)
    {
        int blocks = (int)((capacity + 1023u) / 1024u);
        if (blocks > 148 * 16) blocks = 148 * 16;
        if (blocks < 1) blocks = 1;
        k_ranges<<<blocks, 256, 0, st>>>(tkeys_sorted, ids, depth, w.misc, ranges, keys);
        GS_LAUNCH_CHECK();
    }
    return GS_OK;
}
