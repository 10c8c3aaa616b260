// noalloc.cu -- mlora_apply_noalloc: the fused apply for callers that cannot allocate.
//
// mlora_apply keeps the H values of long segments (the rank-r intermediate of
// segments with 128 or more rows, fp32) in a workspace the pool grows with
// cudaMalloc the first time a batch needs more.  Some callers cannot let a library
// allocate device memory: a serving engine that reserves nearly all of HBM up front
// and serves every buffer from its own allocator, or a loop that must not meet the
// device-wide synchronisation of a cudaMalloc / cudaFree.  For them this entry point
// takes the workspace from a fixed array in the library's own device memory, so a
// call allocates nothing.
//
// When the array is reserved.  Each .cu file of the library is its own module, and
// CUDA loads modules lazily: this file's module (and the array with it) is brought
// onto a device the first time its symbol is looked up there.  mlora_pool_create does
// that look-up for its device (mlora_noalloc_reserve), so the array is reserved when
// the first pool is created on a device -- a call that allocates anyway -- and a later
// mlora_apply_noalloc finds the address cached.  Every GPU that has held a pool keeps
// the array until the process exits.
//
// The array keeps the last call's contents; each call writes every H value it later
// reads, so nothing needs clearing.  Calls whose kernels overlap on the GPU race on
// the one array.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace {

// Largest workspace the entry point can use: grouped rows x max(16, rank bucket of the
// pool's r_max) x 4 bytes must fit (16384 rows for a rank-64 pool, 65536 for rank <= 16).
constexpr size_t kScratchBytes = 4u << 20;

static __device__ __align__(256) float g_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
float *g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per device.  In
// host code `g_scratch` names a host-side stand-in, never the device memory itself.
mlora_status scratch_address(int dev, float **out)
{
    if (dev < 0 || dev >= kMaxDevices) return MLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return MLORA_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<float *>(ptr);
    }
    *out = g_scratch_addr[dev];
    return MLORA_OK;
}

}  // namespace

mlora_status mlora_noalloc_reserve(int dev)
{
    float *unused = nullptr;
    return scratch_address(dev, &unused);
}

extern "C" mlora_status mlora_apply_noalloc(mlora_pool *pool, const mlora_segments *segs,
                                            const void *X, int64_t ldx, void *Y, int64_t ldy,
                                            void *stream)
{
    const int dev = mlora_pool_device(pool);
    if (dev < 0) return MLORA_ERR_INVALID_ARG;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return MLORA_ERR_CUDA;
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) return MLORA_ERR_CUDA;
    float *scratch = nullptr;
    mlora_status st = scratch_address(dev, &scratch);
    if (prev != dev) cudaSetDevice(prev);
    if (st != MLORA_OK) return st;
    return mlora_apply_with_workspace(pool, segs, X, ldx, Y, ldy, stream, scratch, kScratchBytes);
}
