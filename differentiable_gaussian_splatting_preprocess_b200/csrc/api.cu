// Library-level entry points: version, status text, workspace sizing and the
// sticky device status word.

#include <cuda_runtime.h>

#include <atomic>

#include "gs_internal.cuh"

namespace gs {
namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace gs

extern "C" size_t gs_preprocess_ws_bytes(int N);
extern "C" size_t gs_bin_sort_ws_bytes(int N, unsigned capacity, int width, int height);

namespace {
__global__ void k_clear_status(gs::WsHeader* h) { h->status = 0u; }
}  // namespace

extern "C" int gs_version(void) { return (1 << 16) | 0; }

extern "C" unsigned long long gs_launch_count(void) { return gs::g_launches.load(std::memory_order_relaxed); }

extern "C" const char* gs_status_string(int status) {
    switch (status) {
        case GS_OK: return "ok";
        case GS_ERR_INVALID_ARG: return "invalid argument";
        case GS_ERR_CAPACITY: return "pair count exceeds the caller's capacity";
        case GS_ERR_TIMEOUT: return "a bounded device wait gave up";
        case GS_ERR_CUDA: return "CUDA launch or copy failed";
        case GS_ERR_UNIMPLEMENTED: return "not implemented";
        case GS_ERR_OVERFLOW: return "pair count does not fit in 32 bits";
        case GS_ERR_INDEX: return "an index check of the debug build failed";
        default: return "several error flags are set";
    }
}

extern "C" size_t gs_workspace_bytes(int stage, int N, unsigned capacity, int width, int height) {
    if (N < 0 || width < 1 || height < 1) return 0;
    switch (stage) {
        case GS_STAGE_PREPROCESS_FWD: return gs_preprocess_ws_bytes(N);
        case GS_STAGE_BIN_SORT: return gs_bin_sort_ws_bytes(N, capacity, width, height);
        default: return 0;
    }
}

extern "C" int gs_read_status(const void* ws, int* status, void* stream) {
    if (!ws || !status) return GS_ERR_INVALID_ARG;
    unsigned v = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&v, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    *status = (int)v;
    return GS_OK;
}

#ifdef GS_DEBUG
namespace gs {
__device__ DebugState g_debug = {0xFFFFFFFFu, 0xFFFFFFFFu, 0u, 0u};
}  // namespace gs

extern "C" int gs_debug_configure(unsigned n_gauss, unsigned capacity) {
    const gs::DebugState d = {n_gauss, capacity, 0u, 0u};
    if (cudaMemcpyToSymbol(gs::g_debug, &d, sizeof d) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    return GS_OK;
}

extern "C" int gs_debug_read(int* flags, int clear) {
    if (!flags) return GS_ERR_INVALID_ARG;
    gs::DebugState d;
    if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyFromSymbol(&d, gs::g_debug, sizeof d) != cudaSuccess) {
        (void)cudaGetLastError();
        return GS_ERR_CUDA;
    }
    *flags = (int)d.flags;
    if (clear) {
        d.flags = 0u;
        if (cudaMemcpyToSymbol(gs::g_debug, &d, sizeof d) != cudaSuccess) {
            (void)cudaGetLastError();
            return GS_ERR_CUDA;
        }
    }
    return GS_OK;
}
#else
extern "C" int gs_debug_configure(unsigned, unsigned) { return GS_ERR_UNIMPLEMENTED; }

extern "C" int gs_debug_read(int* flags, int) {
    if (flags) *flags = 0;
    return GS_ERR_UNIMPLEMENTED;
}
#endif

extern "C" int gs_clear_status(void* ws, void* stream) {
    if (!ws) return GS_ERR_INVALID_ARG;
    k_clear_status<<<1, 1, 0, (cudaStream_t)stream>>>(reinterpret_cast<gs::WsHeader*>(ws)); gs::note_launch();
    GS_LAUNCH_CHECK();
    return GS_OK;
}
