// noalloc.cu -- pc_modup_noalloc: ModUp without a caller-provided workspace.
//
// pc_modup needs l*N words of device scratch for the coefficient form of c1,
// which the caller normally allocates and hands over with pc_set_workspace.
// Some callers cannot allocate device memory at all: a plugin running inside
// a host framework that owns every device allocation, or a latency-critical
// path where a cudaMalloc (which can synchronise the whole device) is not
// acceptable.  For them this file provides the same operation with its
// scratch in a fixed, statically allocated device array instead.
//
// The array is a file-scope __device__ variable of PC_NOALLOC_SCRATCH_WORDS
// 32-bit words (8 MiB): every GPU on which the library is loaded holds it
// until the process exits.  Host code cannot use the variable's name as a
// device address, so the address is looked up once per device with
// cudaGetSymbolAddress (on the first call made on that device, with that
// device current) and cached.  Every call shares the one array and it keeps
// the previous call's contents; calls whose kernels overlap on the GPU (two
// streams, or two host threads) race on it.  Nothing in it needs clearing:
// each call overwrites the l*N words it reads.
#include <cuda_runtime.h>

#include <mutex>

#include "pc_internal.h"

namespace {

constexpr size_t PC_NOALLOC_SCRATCH_WORDS = (size_t)1 << 21;  // 8 MiB
constexpr int MAX_DEVICES = 128;

}  // namespace

static __device__ __align__(256) uint32_t pc_noalloc_scratch[PC_NOALLOC_SCRATCH_WORDS];

namespace {

std::mutex g_scratch_mu;
void *g_scratch_addr[MAX_DEVICES];

// Device address of pc_noalloc_scratch on `dev` (which must be current).
int scratch_address(int dev, uint32_t **out) {
    if (dev < 0 || dev >= MAX_DEVICES) return PC_E_ARG;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, pc_noalloc_scratch);
        if (e != cudaSuccess || !p) return pc::record_cuda_error(e == cudaSuccess ? cudaErrorUnknown : e);
        g_scratch_addr[dev] = p;
    }
    *out = static_cast<uint32_t *>(g_scratch_addr[dev]);
    return PC_OK;
}

}  // namespace

extern "C" int pc_modup_noalloc(pc_ctx *c, const uint32_t *c1, uint32_t l, uint32_t *ext, pc_stream stream) {
    if (!c || !c1 || !ext || l < 1 || l > c->L) return PC_E_ARG;
    if ((((uintptr_t)c1) | ((uintptr_t)ext)) & 15u) return PC_E_ALIGN;
    if ((size_t)l * c->N > PC_NOALLOC_SCRATCH_WORDS) return PC_E_TOO_BIG;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != c->device && cudaSetDevice(c->device) != cudaSuccess) return pc::record_cuda_error(cudaGetLastError());
    uint32_t *w1 = nullptr;
    int rc = scratch_address(c->device, &w1);
    if (rc == PC_OK) {
        const cudaStream_t s = (cudaStream_t)stream;
        cudaError_t e = pc::launch_row(c, false, c1, w1, 0, l, 1, 0, 0, false, true, s);
        if (e == cudaSuccess) e = pc::launch_colconv(c, 0, w1, 0, ext, 0, l, 1, false, s);
        if (e == cudaSuccess) e = pc::launch_modup_finish(c, c1, ext, l, s);
        if (e != cudaSuccess) rc = pc::record_cuda_error(e);
    }
    if (prev >= 0 && prev != c->device) cudaSetDevice(prev);
    return rc;
}
