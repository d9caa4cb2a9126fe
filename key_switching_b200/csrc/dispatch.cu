// dispatch.cu -- the pc:: launchers: each forwards to the launcher compiled
// for the context's ring degree (kernels.cu, one translation unit per
// degree); and the input-check kernel, which does not depend on the degree.
#include <cuda_runtime.h>

#include "launch.cuh"
#include "ntt.cuh"
#include "pc_internal.h"

namespace pc {

#define PC_NS_DECL(K) namespace n##K {
#define PC_NS_END }
PC_NS_DECL(10)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(11)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(12)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(13)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(14)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(15)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(16)
#include "launchers.inc"
PC_NS_END
PC_NS_DECL(17)
#include "launchers.inc"
PC_NS_END

// call FN of the context's ring degree with the given arguments
#define PC_CASE(K, FN, ...) \
    case K: return n##K::FN(__VA_ARGS__);
#define PC_FORWARD(FN, ...)                                                     \
    switch (c->logN) {                                                          \
        PC_CASE(10, FN, __VA_ARGS__) PC_CASE(11, FN, __VA_ARGS__)               \
        PC_CASE(12, FN, __VA_ARGS__) PC_CASE(13, FN, __VA_ARGS__)               \
        PC_CASE(14, FN, __VA_ARGS__) PC_CASE(15, FN, __VA_ARGS__)               \
        PC_CASE(16, FN, __VA_ARGS__) PC_CASE(17, FN, __VA_ARGS__)               \
        default: return cudaErrorInvalidValue;                                  \
    }

cudaError_t prepare_kernels(pc_ctx *c) { PC_FORWARD(prepare_kernels, c) }

cudaError_t timeline_read(const pc_ctx *c, uint64_t *out) { PC_FORWARD(timeline_read, c, out) }

cudaError_t launch_row(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, bool canonical, bool cm_out, cudaStream_t s, u32 galois,
                       const u32 *mul, u32 *xout, const MacIn *mac) {
    PC_FORWARD(launch_row, c, fwd, in, out, first_prime, nlimbs, Z, zin, zout, canonical, cm_out, s, galois, mul, xout,
               mac)
}

cudaError_t launch_col(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, int scale_mode, cudaStream_t s) {
    PC_FORWARD(launch_col, c, fwd, in, out, first_prime, nlimbs, Z, zin, zout, scale_mode, s)
}

cudaError_t launch_colconv(const pc_ctx *c, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz, u32 l,
                           u32 Z, bool out_cm, cudaStream_t s) {
    PC_FORWARD(launch_colconv, c, mode, src, srcz, out, outz, l, Z, out_cm, s)
}

cudaError_t launch_inner(const pc_ctx *c, bool fused, const u32 *src, size_t srcz, const u32 *c1, size_t c1z,
                         u32 *acc, size_t accz, u32 l, const KeyPack &kp, u32 Z, bool regen, bool pintt,
                         cudaStream_t s, u32 t0, u32 nt, const RotPack *rot) {
    PC_FORWARD(launch_inner, c, fused, src, srcz, c1, c1z, acc, accz, l, kp, Z, regen, pintt, s, t0, nt, rot)
}

cudaError_t launch_moddown_row(const pc_ctx *c, const u32 *U, size_t Uz, const u32 *acc, size_t accz, const u32 *c0,
                               size_t c0z, u32 *out0, u32 *out1, size_t outz, u32 l, u32 Z, cudaStream_t s,
                               const RotPack *rot, const u32 *rx, const u32 *ry, const MacIn *mac) {
    PC_FORWARD(launch_moddown_row, c, U, Uz, acc, accz, c0, c0z, out0, out1, outz, l, Z, s, rot, rx, ry, mac)
}

cudaError_t launch_modup_finish(const pc_ctx *c, const u32 *c1, u32 *ext, u32 l, cudaStream_t s) {
    PC_FORWARD(launch_modup_finish, c, c1, ext, l, s)
}

cudaError_t launch_expand(const pc_ctx *c, const u32 seed[8], u32 l, u32 *out, cudaStream_t s) {
    PC_FORWARD(launch_expand, c, seed, l, out, s)
}

// --------------------------------------------- giant step without rotation
// grid (N / 1024, l, 2), 256 threads of 4 coefficients:
// out[h][i] = sum_{j < n1} d_j[i] (.) bs_j[h][i] mod q_i (64-bit sums, one
// reduction; see MacIn for the operand layout).
__global__ void __launch_bounds__(256) k_mac(Tables T, MacIn m, u32 N, u32 l, u32 *out) {
    const u32 i = blockIdx.y, h = blockIdx.z;
    const PrimeK pk = T.pk[i];
    pdl_wait();
    pdl_trigger();
    const size_t o = (size_t)i * N + 4 * ((size_t)blockIdx.x * 256 + threadIdx.x);
    u64 acc[4];
    const uint4 d0 = *reinterpret_cast<const uint4 *>(m.d + o);
    const uint4 x0 = *reinterpret_cast<const uint4 *>(m.x0[h] + o);
    acc[0] = (u64)d0.x * x0.x; acc[1] = (u64)d0.y * x0.y; acc[2] = (u64)d0.z * x0.z; acc[3] = (u64)d0.w * x0.w;
    for (u32 j = 1; j < m.n1; ++j) {
        const uint4 dj = *reinterpret_cast<const uint4 *>(m.d + j * m.dz + o);
        const uint4 xj = *reinterpret_cast<const uint4 *>(m.xs + (j - 1) * m.xz + h * m.hz + o);
        if (j >= 2) {
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r] = fold64(acc[r], pk.q, pk.q1s);
        }
        acc[0] += (u64)dj.x * xj.x; acc[1] += (u64)dj.y * xj.y; acc[2] += (u64)dj.z * xj.z; acc[3] += (u64)dj.w * xj.w;
    }
    u32 v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) v[r] = shoup(redc64(acc[r], pk.q, pk.qn, pk.q1s), pk.r32, pk.r32s, pk.q);
    *reinterpret_cast<uint4 *>(out + (size_t)h * l * N + o) = make_uint4(v[0], v[1], v[2], v[3]);
}

cudaError_t launch_mac(const pc_ctx *c, const MacIn &m, u32 l, u32 *out, cudaStream_t s) {
    if (c->N < 1024 || m.n1 < 1 || l < 1) return cudaErrorInvalidValue;
    return launch_ex(c, k_mac, dim3(c->N / 1024, l, 2), dim3(256), 0, s, c->tab, m, c->N, l, out);
}

// ------------------------------------------------------------ input checks
// grid (N / 1024, nlimbs, Z), 256 threads of 4 words: OR `bit` into the
// device error word when a residue of limb t is not below its prime.  Limb t
// uses prime: mode 0, global index first + (t mod period); mode 1, the local
// limb (t mod period) at level l; mode 2, global index t mod period.  One
// atomic per CTA at most; reads only the checked buffer.
__global__ void __launch_bounds__(256) k_check(Tables T, const u32 *x, u32 N, size_t zs, int mode, u32 first,
                                               u32 period, u32 l, int bit) {
    const u32 t = blockIdx.y, r = t % period;
    const u32 g = mode == 0 ? first + r : (mode == 1 ? (r < l ? r : T.L + (r - l)) : r);
    const u32 q = T.pk[g].q;
    pdl_wait();
    pdl_trigger();
    const uint4 v = *reinterpret_cast<const uint4 *>(x + blockIdx.z * zs + (size_t)t * N +
                                                     4 * ((size_t)blockIdx.x * 256 + threadIdx.x));
    const bool bad = v.x >= q || v.y >= q || v.z >= q || v.w >= q;
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(T.err, bit);
}

cudaError_t launch_check(const pc_ctx *c, const u32 *x, u32 nlimbs, u32 Z, size_t zs, int mode, u32 first,
                         u32 period, u32 l, int bit, cudaStream_t s) {
    if (nlimbs == 0 || Z == 0 || period == 0 || nlimbs > 65535 || Z > 65535 || c->N < 1024)
        return cudaErrorInvalidValue;
    return launch_ex(c, k_check, dim3(c->N / 1024, nlimbs, Z), dim3(256), 0, s, c->tab, x, c->N, zs, mode, first,
                     period, l, bit);
}

}  // namespace pc
