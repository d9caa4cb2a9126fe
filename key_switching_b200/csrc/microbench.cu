// microbench.cu -- integer-throughput microbenchmark behind pc_microbench.
//
// The key-switching path is bound by the integer pipes, not by HBM or the
// tensor cores, so its roofline needs a measured integer peak.  Each kind runs
// many independent chains per thread (enough instruction-level parallelism to
// hide latency) on every SM:
//   0: Shoup modular multiply by a constant, canonical result (NTT twiddles,
//      basis-conversion constants)          -> modmuls/s
//   1: Montgomery multiply of two variables  -> modmuls/s
//   2: ChaCha12 block function               -> blocks/s
//   3: 32-bit multiply-add (IMAD)            -> instructions/s
//   4: 32-bit add + xor (IADD3 / LOP3)       -> instructions/s
//   5..8: ChaCha12 blocks with rotation subsets on the multiply pipe
//         (mask 1: rot16; 5: rot16+rot8; 3: rot16+rot12; 15: all) -> blocks/s
//   9: ChaCha12, two blocks with interleaved quarter rounds  -> blocks/s
//  10: ChaCha12 with the 16- and 8-bit rotations as byte permutes -> blocks/s
//  11: conditional subtraction min(x, x - q) (the lazy reduction) -> ops/s
//  12: 32-bit rotation by a funnel shift                    -> ops/s
//  13: 32-bit rotation by a byte permute                    -> ops/s
//  14: 64-bit addition                                      -> ops/s
//  15: conditional subtraction by compare and select        -> ops/s
#include <cuda_runtime.h>

#include "chacha.cuh"
#include "modarith.cuh"
#include "pc_internal.h"

namespace pc {

constexpr int MB_CHAINS = 8;
constexpr int MB_THREADS = 256;

template <int MASK>
__device__ __forceinline__ void micro_chacha(u32 x[MB_CHAINS], u32 it, u32 tid, const u32 *mul) {
    ChaRot<MASK> R;
#pragma unroll
    for (int i = 0; i < 4; ++i) R.mul[i] = mul[i];
    u32 k[8], out[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) k[i] = x[i];
    chacha12_block(k, it, tid, 0, out, R);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] ^= out[i] + out[i + 8];
}

template <int KIND>
__global__ void __launch_bounds__(MB_THREADS) k_micro(u32 iters, u32 q, u32 w, u32 ws, u32 qn, u32 *sink) {
    const u32 tid = blockIdx.x * blockDim.x + threadIdx.x;
    u32 x[MB_CHAINS], y[MB_CHAINS];
#pragma unroll
    for (int i = 0; i < MB_CHAINS; ++i) {
        x[i] = (tid * 2654435761u + i * 40503u) % q;
        y[i] = (tid * 40503u + i * 2654435761u) % q;
    }
    u32 acc = 0;
    for (u32 it = 0; it < iters; ++it) {
        if constexpr (KIND == 0) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = shoup(x[i], w, ws, q);
        } else if constexpr (KIND == 1) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) {
                const u64 p = (u64)x[i] * y[i];
                x[i] = redc((u32)p, (u32)(p >> 32), q, qn);
            }
        } else if constexpr (KIND == 2) {
            u32 k[8], out[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) k[i] = x[i];
            chacha12_block(k, it, tid, 0, out);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] ^= out[i] + out[i + 8];
        } else if constexpr (KIND == 10) {
            u32 k[8], out[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) k[i] = x[i];
            chacha12_block(k, it, tid, 0, out, ChaRotPrmt{});
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] ^= out[i] + out[i + 8];
        } else if constexpr (KIND == 9) {
            u32 k[8], o0[16], o1[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) k[i] = x[i];
            chacha12_block2(k, 2 * it, tid, 0, o0, o1);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] ^= o0[i] + o1[i + 8];
        } else if constexpr (KIND == 11) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = red1(x[i] + w, q);
        } else if constexpr (KIND == 12) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = __funnelshift_l(x[i], x[i], 7);
        } else if constexpr (KIND == 13) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = __byte_perm(x[i], x[i], 0x2103);
        } else if constexpr (KIND == 14) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS / 2; ++i) {
                u64 a = ((u64)x[2 * i] << 32) | x[2 * i + 1];
                a += ((u64)y[i] << 32) | w;
                x[2 * i] = (u32)(a >> 32);
                x[2 * i + 1] = (u32)a;
            }
        } else if constexpr (KIND == 15) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) {
                const u32 t = x[i] + w;
                x[i] = t >= q ? t - q : t;
            }
        } else if constexpr (KIND >= 5) {
            constexpr int MASK = KIND == 5 ? 1 : KIND == 6 ? 5 : KIND == 7 ? 3 : 15;
            const u32 mul[4] = {w & 0 | (1u << 16), 1u << 12, 1u << 8, 1u << 7};
            u32 m[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) m[i] = mul[i] ^ (ws & 0x80000000u & qn);  // opaque to the compiler
            micro_chacha<MASK>(x, it, tid, m);
        } else if constexpr (KIND == 3) {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = x[i] * y[i] + w;
        } else {
#pragma unroll
            for (int i = 0; i < MB_CHAINS; ++i) x[i] = (x[i] ^ y[i]) + w;
        }
    }
#pragma unroll
    for (int i = 0; i < MB_CHAINS; ++i) acc ^= x[i];
    if (acc == 0x9e3779b9u) sink[0] = acc;  // keeps the chains live
}

template <int KIND>
static cudaError_t run_micro(int sms, u32 iters, u32 *sink, float *ms) {
    const u32 q = 2147352577u, w = 123456789u % q;
    const u32 ws = (u32)(((u64)w << 32) / q);
    u32 inv = q;
    for (int i = 0; i < 5; ++i) inv *= 2 - q * inv;
    const u32 qn = 0u - inv;
    const int blocks = sms * 8;
    k_micro<KIND><<<blocks, MB_THREADS>>>(iters / 16 + 1, q, w, ws, qn, sink);  // warm-up
    cudaEvent_t a, b;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    cudaEventRecord(a);
    k_micro<KIND><<<blocks, MB_THREADS>>>(iters, q, w, ws, qn, sink);
    cudaEventRecord(b);
    cudaError_t e = cudaEventSynchronize(b);
    cudaEventElapsedTime(ms, a, b);
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e;
}

}  // namespace pc

extern "C" int pc_microbench(int device, int kind, uint32_t iters, double *ops_per_s) {
    using namespace pc;
    if (!ops_per_s || kind < 0 || kind > 15 || iters < 1) return PC_E_ARG;
    if (cudaSetDevice(device) != cudaSuccess) return PC_E_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return PC_E_CUDA;
    u32 *sink = nullptr;
    if (cudaMalloc(&sink, 16) != cudaSuccess) return PC_E_CUDA;
    float ms = 0.f;
    cudaError_t e;
    switch (kind) {
        case 0: e = run_micro<0>(sms, iters, sink, &ms); break;
        case 1: e = run_micro<1>(sms, iters, sink, &ms); break;
        case 2: e = run_micro<2>(sms, iters, sink, &ms); break;
        case 3: e = run_micro<3>(sms, iters, sink, &ms); break;
        case 5: e = run_micro<5>(sms, iters, sink, &ms); break;
        case 6: e = run_micro<6>(sms, iters, sink, &ms); break;
        case 7: e = run_micro<7>(sms, iters, sink, &ms); break;
        case 8: e = run_micro<8>(sms, iters, sink, &ms); break;
        case 9: e = run_micro<9>(sms, iters, sink, &ms); break;
        case 10: e = run_micro<10>(sms, iters, sink, &ms); break;
        case 11: e = run_micro<11>(sms, iters, sink, &ms); break;
        case 12: e = run_micro<12>(sms, iters, sink, &ms); break;
        case 13: e = run_micro<13>(sms, iters, sink, &ms); break;
        case 14: e = run_micro<14>(sms, iters, sink, &ms); break;
        case 15: e = run_micro<15>(sms, iters, sink, &ms); break;
        default: e = run_micro<4>(sms, iters, sink, &ms); break;
    }
    cudaFree(sink);
    if (e != cudaSuccess || ms <= 0.f) return PC_E_CUDA;
    const double threads = (double)sms * 8 * MB_THREADS;
    const double per_iter = kind == 9 ? 2.0 : (kind == 2 || (kind >= 5 && kind <= 10)) ? 1.0 : (double)MB_CHAINS;
    *ops_per_s = threads * per_iter * (double)iters / (ms * 1e-3);
    return PC_OK;
}
