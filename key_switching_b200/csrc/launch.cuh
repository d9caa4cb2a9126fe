// launch.cuh -- the one way libpc launches a kernel (shared by the
// translation units that launch kernels).
#pragma once
#include <cuda_runtime.h>

#include "pc_internal.h"

namespace pc {

// Every launch goes through cudaLaunchKernelEx with programmatic stream
// serialisation (the kernels call pdl_wait before touching data) and, when the
// context has one, an L2 access-policy window that keeps the constant tables
// persisting in L2 while the streamed operands pass through.
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_exc(const pc_ctx *c, unsigned cluster_x, void (*kern)(KArgs...), dim3 grid, dim3 block,
                              size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[3];
    unsigned n = 0;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (c->use_pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (c->l2_window_bytes) {
        attr[n].id = cudaLaunchAttributeAccessPolicyWindow;
        attr[n].val.accessPolicyWindow.base_ptr = c->l2_window_base;
        attr[n].val.accessPolicyWindow.num_bytes = c->l2_window_bytes;
        attr[n].val.accessPolicyWindow.hitRatio = c->l2_hit_ratio;
        attr[n].val.accessPolicyWindow.hitProp = cudaAccessPropertyPersisting;
        attr[n].val.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
static inline cudaError_t launch_ex(const pc_ctx *c, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args... args) {
    return launch_exc(c, 1, kern, grid, block, smem, s, args...);
}

}  // namespace pc
