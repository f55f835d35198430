// vf_concretize_dense_noalloc: the concretising dense back-substitution step for callers that cannot
// allocate device memory.
//
// Who needs it: code whose device memory is owned by another allocator (a host framework's pool that
// forbids raw cudaMalloc), code that runs under a fixed device-memory budget, and code that must not pay
// the device-wide synchronisation that cudaMalloc / cudaFree can imply. Such callers can still provide
// their own inputs and outputs, but not the scratch space that the per-N-tile partial sums and the row
// constants of this step need. Here that scratch is a file-scope __device__ array of fixed size, which
// every GPU that loads this library holds until the process exits.
//
// Nothing in this file allocates: the array is reached through cudaGetSymbolAddress, cleared with
// cudaMemsetAsync and used by the same FFMA contraction and row-sum kernels as the handle-based path.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "vf.h"
#include "vf_internal.cuh"

using namespace vf;

namespace {

// 4 Mi floats (16 MiB): row constants [M] followed by per-N-tile partials [tiles, M].
constexpr long long kScratchFloats = VF_NOALLOC_SCRATCH_FLOATS;
static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

// Device address of g_noalloc_scratch per device. In host code the symbol's name is only a host-side
// stand-in, so the address must be looked up on each device (with that device current) before use. The
// address is cached for the life of the process: a caller that resets a device (cudaDeviceReset) destroys
// the module the array lives in, and must not call this entry point on that device afterwards.
constexpr int kMaxDevices = 64;
float* g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Errors go to the same per-thread message as every other entry point (vf_last_error).
int noalloc_fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    return set_last_error(code, buf);
}

int scratch_for_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return noalloc_fail(VF_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(VF_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_dev[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return noalloc_fail(VF_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev,
                                cudaGetErrorString(e));
        g_scratch_dev[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_dev[dev];
    return VF_OK;
}

}  // namespace

extern "C" {

int vf_concretize_dense_noalloc(const float* lambda, long long lambda_bstride, int R, const float* W, const float* b,
                                const float* centres, float eps, int B, int n_in, int n_out, float* lb, void* stream) {
    if (!lambda || !W || !b || !centres || !lb) return noalloc_fail(VF_ERR_ARG, "NULL pointer");
    if (B < 0 || R < 0 || n_in <= 0 || n_out <= 0 || lambda_bstride < 0)
        return noalloc_fail(VF_ERR_ARG, "bad sizes");
    if (lambda_bstride > 0 && lambda_bstride < (long long)R * n_out)
        return noalloc_fail(VF_ERR_ARG, "lambda_bstride %lld is below one centre's R * n_out = %lld elements",
                            lambda_bstride, (long long)R * n_out);
    if (!std::isfinite(eps) || eps < 0.f) return noalloc_fail(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (B == 0 || R == 0) return VF_OK;
    const long long M = (long long)B * R;
    const int tiles = dense_back_tiles_n(n_in);
    const long long need = M * (1LL + tiles);
    if (need > kScratchFloats)
        return noalloc_fail(VF_ERR_WORKSPACE,
                            "B*R*(1 + ceil(n_in / tile)) = %lld floats exceeds the fixed scratch of %lld floats "
                            "(B*R = %lld rows, %d column tiles); split the rows into smaller calls",
                            need, kScratchFloats, M, tiles);
    float* scratch = nullptr;
    int rc = scratch_for_current_device(&scratch);
    if (rc != VF_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    float* cst = scratch;       // row constants, must start at zero
    float* part = scratch + M;  // per-N-tile partials, fully overwritten by the contraction
    cudaError_t e = cudaMemsetAsync(cst, 0, sizeof(float) * M, s);
    if (e != cudaSuccess) return noalloc_fail(VF_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    const RowRef A{lambda, lambda_bstride, n_out, R, 0};
    e = launch_dense_back(A, Relax{nullptr, 0}, W, b, M, n_out, n_in, PassGeom{0, R}, OUT_CONCRETIZE, nullptr, 0, cst,
                          centres, eps, part, s);
    if (e != cudaSuccess) return noalloc_fail(VF_ERR_CUDA, "contraction launch: %s", cudaGetErrorString(e));
    e = launch_finish_rows(cst, part, tiles, M, lb, s);
    if (e != cudaSuccess) return noalloc_fail(VF_ERR_CUDA, "row-sum launch: %s", cudaGetErrorString(e));
    return VF_OK;
}

}  // extern "C"
