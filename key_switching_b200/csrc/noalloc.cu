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
// device address (in host code it names a host-side stand-in), so
// pc_ctx_create looks the address up once per context, with the context's
// device current, through noalloc_setup below, and the entry point passes
// that address to the kernels.  Every call shares the one array and it keeps
// the previous call's contents; calls whose kernels overlap on the GPU (two
// streams, or two host threads) race on it.  Nothing in it needs clearing:
// each call overwrites the l*N words it reads.
#include <cuda_runtime.h>

#include "pc_internal.h"

namespace {
constexpr size_t PC_NOALLOC_SCRATCH_WORDS = (size_t)1 << 21;  // 8 MiB
}  // namespace

static __device__ __align__(256) uint32_t pc_noalloc_scratch[PC_NOALLOC_SCRATCH_WORDS];

namespace pc {

cudaError_t noalloc_setup(pc_ctx *c) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, pc_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    c->noalloc_scratch = static_cast<uint32_t *>(p);
    return cudaSuccess;
}

}  // namespace pc

extern "C" int pc_modup_noalloc(pc_ctx *c, const uint32_t *c1, uint32_t l, uint32_t *ext, pc_stream stream) {
    if (!c || !c1 || !ext || l < 1 || l > c->L) return PC_E_ARG;
    if ((((uintptr_t)c1) | ((uintptr_t)ext)) & 15u) return PC_E_ALIGN;
    if ((size_t)l * c->N > PC_NOALLOC_SCRATCH_WORDS) return PC_E_TOO_BIG;
    if (!c->noalloc_scratch) return PC_E_ARG;
    pc::DeviceGuard dg(c->device);
    if (!dg.ok) return pc::record_cuda_error(cudaGetLastError());
    uint32_t *w1 = c->noalloc_scratch;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (c->checks & PC_CHECK_INPUTS) e = pc::launch_check(c, c1, l, 1, 0, 1, 0, l, l, PC_ERR_INPUT, s);
    if (e == cudaSuccess) e = pc::launch_row(c, false, c1, w1, 0, l, 1, 0, 0, false, true, s);
    if (e == cudaSuccess) e = pc::launch_colconv(c, 0, w1, 0, ext, 0, l, 1, false, s);
    if (e == cudaSuccess) e = pc::launch_modup_finish(c, c1, ext, l, s);
    return e == cudaSuccess ? PC_OK : pc::record_cuda_error(e);
}
