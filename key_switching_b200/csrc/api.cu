// api.cu -- libpc host side: parameter checks, device constant tables, the
// extern "C" entry points declared in include/pc.h, and argument marshalling
// into the kernels of kernels.cu.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "pc_internal.h"

using pc::u32;
using pc::u64;

namespace {

thread_local cudaError_t g_last_cuda = cudaSuccess;

int cuda_fail(cudaError_t e) {
    g_last_cuda = e;
    return PC_E_CUDA;
}

// ---------------------------------------------------------------- host math

u32 mulm(u32 a, u32 b, u32 q) { return (u32)(((u64)a * b) % q); }

u32 powm(u32 a, u64 e, u32 q) {
    u64 r = 1, x = a % q;
    for (; e; e >>= 1) {
        if (e & 1) r = r * x % q;
        x = x * x % q;
    }
    return (u32)(r % q);
}

u32 invm(u32 a, u32 q) { return powm(a, q - 2, q); }

u32 shoup_of(u32 w, u32 q) { return (u32)(((u64)w << 32) / q); }

// strong-probable-prime test to the bases 2, 3, 5, 7, 11: exact for every
// n < 2,152,302,898,747 (Jaeschke 1993), so for all 32-bit n
bool is_prime32(u32 n) {
    if (n < 2) return false;
    static const u32 small[] = {2, 3, 5, 7, 11, 13};
    for (u32 p : small) {
        if (n == p) return true;
        if (n % p == 0) return false;
    }
    u32 d = n - 1;
    int s = 0;
    while (!(d & 1)) { d >>= 1; ++s; }
    static const u32 bases[] = {2, 3, 5, 7, 11};
    for (u32 a : bases) {
        u32 x = powm(a, d, n);
        if (x == 1 || x == n - 1) continue;
        bool witness = true;
        for (int i = 1; i < s && witness; ++i) {
            x = mulm(x, x, n);
            if (x == n - 1) witness = false;
        }
        if (witness) return false;
    }
    return true;
}

// The smallest primitive 2N-th root of unity mod q.  Find one root c (a
// power x^((q-1)/2N) with c^N = -1), then every primitive 2N-th root is c^k
// for odd k < 2N; take the minimum over them.
u32 min_primitive_root_2n(u32 q, u32 logN) {
    const u64 N = 1ull << logN, twoN = 2 * N;
    if ((q - 1) % twoN) return 0;
    u32 c = 0;
    for (u32 x = 2; x < q && !c; ++x) {
        u32 y = powm(x, (q - 1) / twoN, q);
        if (powm(y, N, q) == q - 1) c = y;
    }
    if (!c) return 0;
    const u32 c2 = mulm(c, c, q);
    u32 best = c, r = c;
    for (u64 k = 1; k < N; ++k) {
        r = mulm(r, c2, q);
        if (r < best) best = r;
    }
    return best;
}

u32 brv(u32 x, u32 bits) {
    u32 r = 0;
    for (u32 i = 0; i < bits; ++i) r |= ((x >> i) & 1u) << (bits - 1 - i);
    return r;
}

// -u^-1 mod 2^32 for odd u (Newton iteration)
u32 neg_inv32(u32 u) {
    u32 x = u;  // correct to 3 bits
    for (int i = 0; i < 5; ++i) x *= 2 - u * x;
    return 0u - x;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

using pc::DeviceGuard;

// workspace regions for B ciphertexts at level l (words)
struct Layout {
    size_t w1, t, acc, u, x, total;  // offsets and total, in words
    size_t w1z, tz, accz, uz, xz;    // per-ciphertext strides
};
Layout layout(const pc_ctx *c, u32 l, u32 B) {
    Layout L{};
    const size_t N = c->N, ll = l + c->alpha, beta = (l + c->alpha - 1) / c->alpha;
    L.w1z = l * N;
    L.tz = beta * ll * N;
    L.accz = 2 * ll * N;
    L.uz = 2 * (size_t)l * N;
    L.w1 = 0;
    L.t = L.w1 + B * L.w1z;
    L.acc = L.t + B * L.tz;
    L.u = L.acc + B * L.accz;
    // X: c1 as the ModUp read it (rotated, or relinearisation's d2), for the
    // own-digit limbs of the inner product
    L.xz = l * N;
    L.x = L.u + B * L.uz;
    L.total = L.x + B * L.xz;
    return L;
}

int check_ksk(const pc_ctx *c, const pc_ksk *k) {
    if (!k || !k->b) return PC_E_ARG;
    if (!aligned16(k->b) || (k->a && !aligned16(k->a))) return PC_E_ALIGN;
    (void)c;
    return PC_OK;
}

void seed_words(const uint8_t s[32], u32 out[8]) {
    for (int w = 0; w < 8; ++w)
        out[w] = (u32)s[4 * w] | ((u32)s[4 * w + 1] << 8) | ((u32)s[4 * w + 2] << 16) |
                 ((u32)s[4 * w + 3] << 24);
}

void prof_release(pc_ctx *c) {
    if (!c->prof_ev) return;
    for (size_t i = 0; i < (size_t)c->prof_max * (PC_PROFILE_STAGES + 1); ++i) cudaEventDestroy(c->prof_ev[i]);
    delete[] c->prof_ev;
    c->prof_ev = nullptr;
    c->prof_max = c->prof_used = 0;
}

// PC_CHECK_INPUTS: before a call runs, a kernel checks that every residue
// it reads is canonical and records a violation in the device error word.
cudaError_t check_limbs(const pc_ctx *c, const u32 *x, u32 nlimbs, u32 Z, size_t zs, int mode, u32 first,
                               u32 period, u32 l, int bit, cudaStream_t s) {
    if (!(c->checks & PC_CHECK_INPUTS) || !x) return cudaSuccess;
    return pc::launch_check(c, x, nlimbs, Z, zs, mode, first, period, l, bit, s);
}
// a ciphertext-like input: Z slices of nlimbs limbs, limb t mod l on q_t
cudaError_t check_ct(const pc_ctx *c, const u32 *x, u32 nlimbs, u32 l, u32 Z, size_t zs, cudaStream_t s) {
    return check_limbs(c, x, nlimbs, Z, zs, 1, 0, l, l, PC_ERR_INPUT, s);
}
// both halves of n keys ([dnum][L+alpha][N], global prime of limb t = t mod (L+alpha))
cudaError_t check_keys(const pc_ctx *c, const pc_ksk *k, u32 n, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    for (u32 i = 0; i < n && e == cudaSuccess; ++i) {
        e = check_limbs(c, k[i].b, c->dnum * c->NP, 1, 0, 2, 0, c->NP, 0, PC_ERR_KEY, s);
        if (e == cudaSuccess) e = check_limbs(c, k[i].a, c->dnum * c->NP, 1, 0, 2, 0, c->NP, 0, PC_ERR_KEY, s);
    }
    return e;
}

}  // namespace

namespace pc {
int record_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace pc

extern "C" {

int pc_gen_primes(uint32_t logN, uint32_t bits, uint32_t count, uint32_t *out) {
    if (!out || logN < 1 || logN > 30 || bits < 2 || bits > 31) return PC_E_ARG;
    const u64 twoN = 2ull << logN;
    u64 k = (((u64)1 << bits) - 1) / twoN;
    u32 found = 0;
    while (found < count) {
        if (k == 0) return PC_E_ARG;
        const u64 cand = k * twoN + 1;
        if (is_prime32((u32)cand)) out[found++] = (u32)cand;
        --k;
    }
    return PC_OK;
}

int pc_ctx_create(const pc_params *P, int device, pc_ctx **out) {
    if (!P || !out || !P->q || !P->p) return PC_E_ARG;
    *out = nullptr;
    if (P->logN < 10 || P->logN > 17) return PC_E_ARG;
    if (P->L < 1 || P->L > (u32)pc::MAX_L || P->alpha < 1 || P->alpha > (u32)pc::MAX_ALPHA) return PC_E_ARG;
    if (P->dnum != (P->L + P->alpha - 1) / P->alpha) return PC_E_ARG;
    const u32 N = 1u << P->logN, NP = P->L + P->alpha;
    std::vector<u32> pr(NP);
    for (u32 i = 0; i < P->L; ++i) pr[i] = P->q[i];
    for (u32 i = 0; i < P->alpha; ++i) pr[P->L + i] = P->p[i];
    for (u32 i = 0; i < NP; ++i) {
        if (pr[i] >= (1u << 31) || pr[i] < 3 || (pr[i] - 1) % (2 * N) || !is_prime32(pr[i])) return PC_E_PRIME;
        for (u32 j = 0; j < i; ++j)
            if (pr[j] == pr[i]) return PC_E_PRIME;
    }
    DeviceGuard dg(device);
    if (!dg.ok) return cuda_fail(cudaGetLastError());

    pc_ctx *c = new (std::nothrow) pc_ctx();
    if (!c) return PC_E_ARG;
    c->device = device;
    c->logN = P->logN;
    c->N = N;
    c->L = P->L;
    c->alpha = P->alpha;
    c->dnum = P->dnum;
    c->NP = NP;
    for (u32 i = 0; i < NP; ++i) c->primes[i] = pr[i];
    cudaError_t e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) { delete c; return cuda_fail(e); }

    const u32 logC = (P->logN - 4 < 8) ? P->logN - 4 : 8, logR = P->logN - logC;
    const u32 C = 1u << logC, R = 1u << logR;
    const u32 L = P->L, A = P->alpha, D = P->dnum;

    // host images of every table
    std::vector<pc::PrimeK> pk(NP);
    std::vector<uint2> colF((size_t)NP * R), colI((size_t)NP * R);
    std::vector<uint2> rowF((size_t)NP * N), rowI((size_t)NP * N);
    std::vector<uint2> upScale((size_t)A * L, make_uint2(0, 0));
    std::vector<u32> upConv((size_t)D * A * NP * A, 0);
    std::vector<uint2> downScale(A);
    std::vector<u32> downConv((size_t)L * A);
    std::vector<uint2> pInv(L);
    std::vector<u32> pw(N), pwi(N);

    for (u32 g = 0; g < NP; ++g) {
        const u32 q = pr[g];
        const u32 psi = min_primitive_root_2n(q, P->logN);
        if (!psi) { delete c; return PC_E_PRIME; }
        c->psi[g] = psi;
        const u32 psii = invm(psi, q);
        pw[0] = 1;
        pwi[0] = 1;
        for (u32 k = 1; k < N; ++k) {
            pw[k] = mulm(pw[k - 1], psi, q);
            pwi[k] = mulm(pwi[k - 1], psii, q);
        }
        auto rev = [&](const std::vector<u32> &t, u32 k) { return t[brv(k, P->logN)]; };
        // re-laid position of natural table entry k (see TwRow in ntt.cuh)
        auto relay = [](u32 k) -> u32 {
            if (k == 0) return 0;
            u32 s = 0;
            while ((2u << s) <= k) ++s;
            const u32 i = k - (1u << s), u = s & 3u, s0 = s - u;
            return (1u << s) + ((i & ((1u << u) - 1)) << s0) + (i >> u);
        };
        for (u32 k = 0; k < R; ++k) {
            const u32 a = rev(pw, k), b = rev(pwi, k);
            colF[(size_t)g * R + relay(k)] = make_uint2(a, shoup_of(a, q));
            colI[(size_t)g * R + relay(k)] = make_uint2(b, shoup_of(b, q));
        }
        for (u32 r = 0; r < R; ++r) {
            const size_t base = (size_t)g * N + (size_t)r * C;
            rowF[base] = make_uint2(0, 0);
            rowI[base] = make_uint2(0, 0);
            for (u32 k = 1; k < C; ++k) {
                // natural entry k = 2^s + i holds psi_rev[(R + r) 2^s + i]
                u32 s = 0;
                while ((2u << s) <= k) ++s;
                const u32 i = k - (1u << s);
                const u32 idx = (R + r) * (1u << s) + i;
                const u32 a = rev(pw, idx), b = rev(pwi, idx);
                rowF[base + relay(k)] = make_uint2(a, shoup_of(a, q));
                rowI[base + relay(k)] = make_uint2(b, shoup_of(b, q));
            }
        }
        pc::PrimeK &K = pk[g];
        memset(&K, 0, sizeof(K));
        K.q = q;
        K.qn = neg_inv32(q);
        K.q1s = (u32)((1ull << 32) / q);
        K.r32 = (u32)((1ull << 32) % q);
        K.r32s = shoup_of(K.r32, q);
        K.r64 = mulm(K.r32, K.r32, q);
        K.r64s = shoup_of(K.r64, q);
        K.ninv = invm(N % q, q);
        K.ninvs = shoup_of(K.ninv, q);
    }
    // ModUp: digit j of size d covers q_{j A} .. q_{j A + d - 1}
    for (u32 j = 0; j < D; ++j) {
        for (u32 d = 1; d <= A; ++d) {
            const u32 lo = j * A;
            if (lo + d > L) continue;
            for (u32 k = 0; k < d; ++k) {
                const u32 i = lo + k, qi = pr[i];
                u32 dh = 1;
                for (u32 m = 0; m < d; ++m)
                    if (m != k) dh = mulm(dh, pr[lo + m] % qi, qi);
                const u32 s = mulm(invm(N % qi, qi), invm(dh, qi), qi);
                upScale[(size_t)(d - 1) * L + i] = make_uint2(s, shoup_of(s, qi));
                for (u32 g = 0; g < NP; ++g) {
                    const u32 t = pr[g];
                    u32 dt = 1;
                    for (u32 m = 0; m < d; ++m)
                        if (m != k) dt = mulm(dt, pr[lo + m] % t, t);
                    upConv[(((size_t)j * A + (d - 1)) * NP + g) * A + k] = mulm(dt, (u32)((1ull << 32) % t), t);
                }
            }
        }
    }
    // ModDown
    for (u32 k = 0; k < A; ++k) {
        const u32 p = pr[L + k];
        u32 ph = 1;
        for (u32 m = 0; m < A; ++m)
            if (m != k) ph = mulm(ph, pr[L + m] % p, p);
        const u32 s = mulm(invm(N % p, p), invm(ph, p), p);
        downScale[k] = make_uint2(s, shoup_of(s, p));
    }
    for (u32 i = 0; i < L; ++i) {
        const u32 qi = pr[i];
        u32 Pm = 1;
        for (u32 k = 0; k < A; ++k) {
            Pm = mulm(Pm, pr[L + k] % qi, qi);
            u32 ph = 1;
            for (u32 m = 0; m < A; ++m)
                if (m != k) ph = mulm(ph, pr[L + m] % qi, qi);
            downConv[(size_t)i * A + k] = mulm(ph, (u32)((1ull << 32) % qi), qi);
        }
        const u32 pi = invm(Pm, qi);
        pInv[i] = make_uint2(pi, shoup_of(pi, qi));
    }

    // one device allocation, 256-byte aligned sub-buffers
    struct Piece { const void *src; size_t bytes; size_t off; };
    std::vector<Piece> pieces = {
        {pk.data(), pk.size() * sizeof(pc::PrimeK), 0},
        {colF.data(), colF.size() * sizeof(uint2), 0},
        {colI.data(), colI.size() * sizeof(uint2), 0},
        {rowF.data(), rowF.size() * sizeof(uint2), 0},
        {rowI.data(), rowI.size() * sizeof(uint2), 0},
        {upScale.data(), upScale.size() * sizeof(uint2), 0},
        {upConv.data(), upConv.size() * sizeof(u32), 0},
        {downScale.data(), downScale.size() * sizeof(uint2), 0},
        {downConv.data(), downConv.size() * sizeof(u32), 0},
        {pInv.data(), pInv.size() * sizeof(uint2), 0},
        {nullptr, 256, 0},  // device error word
    };
    size_t total = 0;
    for (auto &p : pieces) {
        p.off = total;
        total += (p.bytes + 255) & ~(size_t)255;
    }
    void *blk = nullptr;
    e = cudaMalloc(&blk, total);
    if (e != cudaSuccess) { delete c; return cuda_fail(e); }
    for (auto &p : pieces) {
        if (p.src) e = cudaMemcpy((char *)blk + p.off, p.src, p.bytes, cudaMemcpyHostToDevice);
        else e = cudaMemset((char *)blk + p.off, 0, p.bytes);
        if (e != cudaSuccess) { cudaFree(blk); delete c; return cuda_fail(e); }
    }
    auto at = [&](int i) { return (char *)blk + pieces[i].off; };
    c->dev_block = blk;
    c->dev_bytes = total;
    pc::Tables &T = c->tab;
    T.pk = (const pc::PrimeK *)at(0);
    T.colF = (const uint2 *)at(1);
    T.colI = (const uint2 *)at(2);
    T.rowF = (const uint2 *)at(3);
    T.rowI = (const uint2 *)at(4);
    T.upScale = (const uint2 *)at(5);
    T.upConv = (const u32 *)at(6);
    T.downScale = (const uint2 *)at(7);
    T.downConv = (const u32 *)at(8);
    T.pInv = (const uint2 *)at(9);
    T.err = (int *)at(10);
    T.L = L;
    T.alpha = A;
    T.dnum = D;
    T.NP = NP;
    e = pc::prepare_kernels(c);
    if (e != cudaSuccess) { cudaFree(blk); delete c; return cuda_fail(e); }
    // the device address of pc_modup_noalloc's static scratch (device current)
    e = pc::noalloc_setup(c);
    if (e != cudaSuccess) { cudaFree(blk); delete c; return cuda_fail(e); }
    // Launch attributes.  Programmatic dependent launch lets each kernel stage
    // its tables while its predecessor drains.  Opt-in (PC_L2_PERSIST=1 at
    // context creation): an access-policy window marks the constant tables
    // persisting in L2 so the streamed keys and ciphertexts do not evict them;
    // that raises the process's persisting-L2 limit, which other kernels of
    // the process then share, so it is off unless asked for.
    c->use_pdl = getenv("PC_NO_PDL") ? 0 : 1;
    {
        int lo_pri = 0, hi_pri = 0;
        cudaDeviceGetStreamPriorityRange(&lo_pri, &hi_pri);
        e = cudaStreamCreateWithPriority(&c->aux, cudaStreamNonBlocking, hi_pri);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->d2h, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_start, cudaEventDisableTiming);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&c->ev_in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_done[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_out[i], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) { cudaFree(blk); delete c; return cuda_fail(e); }
        c->overlap = getenv("PC_NO_OVERLAP") ? 0 : 1;
    }
    int max_persist = 0, max_window = 0;
    cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, device);
    cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, device);
    const char *l2p = getenv("PC_L2_PERSIST");
    if (l2p && l2p[0] == '1' && max_persist > 0 && max_window > 0) {
        size_t want = total < (size_t)max_persist ? total : (size_t)max_persist;
        size_t cur = 0;
        cudaDeviceGetLimit(&cur, cudaLimitPersistingL2CacheSize);
        if (cur < want && cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, want) != cudaSuccess) {
            cudaGetLastError();
            want = cur;
        }
        if (want > 0) {
            c->l2_window_base = blk;
            c->l2_window_bytes = total < (size_t)max_window ? total : (size_t)max_window;
            const double r = (double)want / (double)c->l2_window_bytes;
            c->l2_hit_ratio = r >= 1.0 ? 1.0f : (float)r;
        }
    }
    *out = c;
    return PC_OK;
}

void pc_ctx_destroy(pc_ctx *c) {
    if (!c) return;
    DeviceGuard dg(c->device);
    prof_release(c);
    if (c->aux) cudaStreamDestroy(c->aux);
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->ev_join) cudaEventDestroy(c->ev_join);
    if (c->h2d) cudaStreamDestroy(c->h2d);
    if (c->d2h) cudaStreamDestroy(c->d2h);
    for (cudaEvent_t ev : {c->ev_start, c->ev_in[0], c->ev_in[1], c->ev_done[0], c->ev_done[1], c->ev_out[0],
                           c->ev_out[1]})
        if (ev) cudaEventDestroy(ev);
    if (c->cap) {  // a capture left open
        cudaGraph_t g = nullptr;
        if (cudaStreamEndCapture(c->cap, &g) == cudaSuccess && g) cudaGraphDestroy(g);
        cudaStreamDestroy(c->cap);
    }
    if (c->dev_block) cudaFree(c->dev_block);
    delete c;
}

uint32_t pc_psi(const pc_ctx *c, uint32_t g) { return (c && g < c->NP) ? c->psi[g] : 0; }

size_t pc_workspace_bytes(const pc_ctx *c, uint32_t l, uint32_t B) {
    if (!c || l < 1 || l > c->L || B < 1) return 0;
    return layout(c, l, B).total * sizeof(u32);
}

// pc_keyswitch_host: the key switch's workspace, then two staging slots of
// one ciphertext in and one out ([2][l][N] each)
static size_t host_ws_words(const pc_ctx *c, u32 l) { return layout(c, l, 1).total + 8 * (size_t)l * c->N; }

size_t pc_host_workspace_bytes(const pc_ctx *c, uint32_t l) {
    if (!c || l < 1 || l > c->L) return 0;
    return host_ws_words(c, l) * sizeof(u32);
}

int pc_set_workspace(pc_ctx *c, void *dev, size_t bytes) {
    if (!c) return PC_E_ARG;
    if (dev && ((uintptr_t)dev & 255u)) return PC_E_ALIGN;
    c->ws = dev;
    c->ws_bytes = dev ? bytes : 0;
    return PC_OK;
}

int pc_ntt_fwd(pc_ctx *c, uint32_t *x, uint32_t first_prime, uint32_t nlimbs, uint32_t batch,
               pc_stream stream) {
    if (!c || !x || nlimbs < 1 || batch < 1 || first_prime + nlimbs > c->NP || batch > 65535) return PC_E_ARG;
    if (!aligned16(x)) return PC_E_ALIGN;
    DeviceGuard dg(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t z = (size_t)nlimbs * c->N;
    if (cudaError_t e = check_limbs(c, x, nlimbs, batch, z, 0, first_prime, nlimbs, 0, PC_ERR_INPUT, s))
        return cuda_fail(e);
    cudaError_t e = pc::launch_col(c, true, x, x, first_prime, nlimbs, batch, z, z, 0, s);
    if (e == cudaSuccess) e = pc::launch_row(c, true, x, x, first_prime, nlimbs, batch, z, z, true, false, s);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_ntt_inv(pc_ctx *c, uint32_t *x, uint32_t first_prime, uint32_t nlimbs, uint32_t batch,
               pc_stream stream) {
    if (!c || !x || nlimbs < 1 || batch < 1 || first_prime + nlimbs > c->NP || batch > 65535) return PC_E_ARG;
    if (!aligned16(x)) return PC_E_ALIGN;
    DeviceGuard dg(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t z = (size_t)nlimbs * c->N;
    if (cudaError_t e = check_limbs(c, x, nlimbs, batch, z, 0, first_prime, nlimbs, 0, PC_ERR_INPUT, s))
        return cuda_fail(e);
    cudaError_t e = pc::launch_row(c, false, x, x, first_prime, nlimbs, batch, z, z, false, false, s);
    if (e == cudaSuccess) e = pc::launch_col(c, false, x, x, first_prime, nlimbs, batch, z, z, 1, s);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

static int need_ws(const pc_ctx *c, u32 l, u32 B) {
    if (!c->ws || c->ws_bytes < layout(c, l, B).total * sizeof(u32)) return PC_E_WORKSPACE;
    return PC_OK;
}

int pc_modup(pc_ctx *c, const uint32_t *c1, uint32_t l, uint32_t *ext, pc_stream stream) {
    if (!c || !c1 || !ext || l < 1 || l > c->L) return PC_E_ARG;
    if (!aligned16(c1) || !aligned16(ext)) return PC_E_ALIGN;
    if (int r = need_ws(c, l, 1)) return r;
    DeviceGuard dg(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const Layout Lw = layout(c, l, 1);
    u32 *w1 = (u32 *)c->ws + Lw.w1;
    cudaError_t e = check_ct(c, c1, l, l, 1, 0, s);
    if (e == cudaSuccess) e = pc::launch_row(c, false, c1, w1, 0, l, 1, 0, 0, false, true, s);
    if (e == cudaSuccess) e = pc::launch_colconv(c, 0, w1, 0, ext, 0, l, 1, false, s);
    if (e == cudaSuccess) e = pc::launch_modup_finish(c, c1, ext, l, s);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_keyswitch_inner(pc_ctx *c, const uint32_t *ext, uint32_t l, const pc_ksk *k, uint32_t *acc,
                       pc_stream stream) {
    if (!c || !ext || !acc || l < 1 || l > c->L) return PC_E_ARG;
    if (int r = check_ksk(c, k)) return r;
    if (!aligned16(ext) || !aligned16(acc)) return PC_E_ALIGN;
    DeviceGuard dg(c->device);
    pc::KeyPack kp{};
    kp.b[0] = k->b;
    kp.a[0] = k->a;
    seed_words(k->seed, kp.seed[0]);
    const cudaStream_t s = (cudaStream_t)stream;
    const u32 beta = (l + c->alpha - 1) / c->alpha, ll = l + c->alpha;
    cudaError_t e = check_limbs(c, ext, beta * ll, 1, 0, 1, 0, ll, l, PC_ERR_INPUT, s);
    if (e == cudaSuccess) e = check_keys(c, k, 1, s);
    if (e == cudaSuccess)
        e = pc::launch_inner(c, false, ext, 0, nullptr, 0, acc, 0, l, kp, 1, k->a == nullptr, false, s);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_moddown(pc_ctx *c, const uint32_t *acc, uint32_t l, uint32_t *out, pc_stream stream) {
    if (!c || !acc || !out || l < 1 || l > c->L) return PC_E_ARG;
    if (!aligned16(acc) || !aligned16(out)) return PC_E_ALIGN;
    if (int r = need_ws(c, l, 1)) return r;
    DeviceGuard dg(c->device);
    cudaStream_t s = (cudaStream_t)stream;
    const Layout Lw = layout(c, l, 1);
    u32 *wacc = (u32 *)c->ws + Lw.acc, *wu = (u32 *)c->ws + Lw.u;
    const size_t N = c->N, ll = l + c->alpha;
    cudaError_t e = check_limbs(c, acc, 2 * (u32)ll, 1, 0, 1, 0, (u32)ll, l, PC_ERR_INPUT, s);
    // special-prime limbs of both halves: inverse row pass into the workspace
    if (e == cudaSuccess)
        e = pc::launch_row(c, false, acc + l * N, wacc + l * N, c->L, c->alpha, 2, ll * N, ll * N, false, true, s);
    if (e == cudaSuccess) e = pc::launch_colconv(c, 1, wacc, 2 * ll * N, wu, 2 * l * N, l, 1, true, s);
    if (e == cudaSuccess) e = pc::launch_moddown_row(c, wu, 0, acc, 0, nullptr, 0, out, out + l * N, 0, l, 1, s);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

// How the kernels read a key switch's inputs.  galois != 1 (single
// rotation): the automorphism X -> X^galois is applied to c1 (ModUp input)
// and c0 as they are read.  hoist (hoisted rotations): slice z of the batch
// applies X -> X^hoist[z] to the extended limbs of one shared ModUp output
// and to c0.  mul: c1 is the slot-wise product c1 * mul (relinearisation's
// d2); rx, ry: the tensor terms d0, d1 of ciphertexts rx, ry are added to the
// outputs instead of c0.
// mac: c1 and c0 are halves 1 and 0 of the giant-step operand W of a linear
// transform (formed from the baby steps and diagonals as they are read), and
// the results are added to the outputs.
struct KsInput {
    u32 galois = 1;
    const u32 *hoist = nullptr;
    const u32 *mul = nullptr, *rx = nullptr, *ry = nullptr;
    const pc::MacIn *mac = nullptr;
};

// x^-1 mod 2N for odd x (Newton iteration on the 2-adic inverse).
static u32 inv_mod_2n(u32 x, u32 N) {
    u32 y = x;  // x * x = 1 mod 8
    for (int i = 0; i < 5; ++i) y *= 2u - x * y;
    return y & (2u * N - 1u);
}

static bool galois_ok(const pc_ctx *c, u32 g) { return (g & 1u) && g < 2u * c->N; }

// events of an instrumented call, or null (measurement only)
static cudaEvent_t *profile_slot(pc_ctx *c) {
    if (c->prof_ev && c->prof_used < c->prof_max && (c->prof_seen++ % c->prof_every) == 0)
        return c->prof_ev + (size_t)(c->prof_used++) * (PC_PROFILE_STAGES + 1);
    return nullptr;
}

// c1 is read transformed by the ModUp row kernel, which then stores that
// transformed copy in the workspace for the inner product's own-digit limbs
static bool c1_transformed(const KsInput &in) { return in.galois != 1 || in.mul || in.mac; }

// ModUp up to the column-pass output T in the workspace (laid out for Blay
// ciphertexts): inverse row pass of c1 (through the input transform), then
// the conversion kernel.
static cudaError_t ks_modup(pc_ctx *c, const u32 *c1, size_t cz, u32 l, u32 B, u32 Blay, const KsInput &in,
                            cudaStream_t s, cudaEvent_t *ev) {
    const Layout Lw = layout(c, l, Blay);
    u32 *ws = (u32 *)c->ws;
    auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };
    mark(0);
    cudaError_t e = pc::launch_row(c, false, c1, ws + Lw.w1, 0, l, B, cz, Lw.w1z, false, true, s, in.galois, in.mul,
                                   c1_transformed(in) ? ws + Lw.x : nullptr, in.mac);
    mark(1);
    if (e == cudaSuccess) e = pc::launch_colconv(c, 0, ws + Lw.w1, Lw.w1z, ws + Lw.t, Lw.tz, l, B, true, s);
    mark(2);
    return e;
}

// Inner products, ModDown and the output combination of B slices, from T in
// the workspace (laid out for Blay ciphertexts; one T shared by every slice
// when hoisting).  Inputs of slice z at stride cz, outputs at stride oz.
static cudaError_t ks_finish(pc_ctx *c, const u32 *c0, const u32 *c1, size_t cz, u32 l, const pc_ksk *keys, u32 B,
                             u32 Blay, u32 *o0, u32 *o1, size_t oz, const KsInput &in, cudaStream_t s,
                             cudaEvent_t *ev) {
    const Layout Lw = layout(c, l, Blay);
    u32 *ws = (u32 *)c->ws;
    u32 *wt = ws + Lw.t, *wacc = ws + Lw.acc, *wu = ws + Lw.u;
    const size_t tz = in.hoist ? 0 : Lw.tz;
    const bool regen = keys[0].a == nullptr;
    auto mark = [&](int i) { if (ev) cudaEventRecord(ev[i], s); };
    cudaError_t e = cudaSuccess;
    // own-digit limbs: c1 itself, or the transformed copy ks_modup stored
    const u32 *own = c1_transformed(in) ? ws + Lw.x : c1;
    const size_t ownz = c1_transformed(in) ? Lw.xz : cz;
    auto rotpack = [&](u32 b0, u32 nb) {
        pc::RotPack rp{};
        for (int z = 0; z < pc::KEYS_PER_LAUNCH; ++z) rp.galois[z] = rp.ginv[z] = 1;
        for (u32 z = 0; z < nb; ++z) {
            rp.galois[z] = in.hoist ? in.hoist[b0 + z] : in.galois;
            rp.ginv[z] = inv_mod_2n(rp.galois[z], c->N);
        }
        return rp;
    };
    // The ModDown branch needs only the special-prime accumulators: when not
    // instrumented, those inner products run first on the high-priority
    // internal stream, followed there by the ModDown conversion kernel, while
    // the ciphertext-prime inner products run on the caller's stream; the
    // final kernel joins both.
    const bool fork = c->overlap && !ev;
    auto inner = [&](cudaStream_t st, u32 t0, u32 nt) {
        for (u32 b0 = 0; e == cudaSuccess && b0 < B; b0 += pc::KEYS_PER_LAUNCH) {
            const u32 nb = (B - b0 < (u32)pc::KEYS_PER_LAUNCH) ? B - b0 : (u32)pc::KEYS_PER_LAUNCH;
            pc::KeyPack kp{};
            for (u32 i = 0; i < nb; ++i) {
                kp.b[i] = keys[b0 + i].b;
                kp.a[i] = keys[b0 + i].a;
                seed_words(keys[b0 + i].seed, kp.seed[i]);
            }
            const pc::RotPack rp = rotpack(b0, nb);
            e = pc::launch_inner(c, true, wt + b0 * tz, tz, own + b0 * ownz, ownz, wacc + b0 * Lw.accz, Lw.accz, l,
                                 kp, nb, regen, true, st, t0, nt, in.hoist ? &rp : nullptr);
        }
    };
    if (fork) {
        e = cudaEventRecord(c->ev_fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(c->aux, c->ev_fork, 0);
        inner(c->aux, l, c->alpha);
        if (e == cudaSuccess) e = pc::launch_colconv(c, 1, wacc, Lw.accz, wu, Lw.uz, l, B, true, c->aux);
        if (e == cudaSuccess) e = cudaEventRecord(c->ev_join, c->aux);
        inner(s, 0, l);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, c->ev_join, 0);
    } else {
        inner(s, 0, 0);
        mark(3);
        if (e == cudaSuccess) e = pc::launch_colconv(c, 1, wacc, Lw.accz, wu, Lw.uz, l, B, true, s);
    }
    mark(4);
    const bool rot = in.hoist || in.galois != 1;
    if (rot && B > (u32)pc::KEYS_PER_LAUNCH) e = cudaErrorInvalidValue;
    const pc::RotPack rp = rotpack(0, B < (u32)pc::KEYS_PER_LAUNCH ? B : (u32)pc::KEYS_PER_LAUNCH);
    if (e == cudaSuccess)
        e = pc::launch_moddown_row(c, wu, Lw.uz, wacc, Lw.accz, in.rx ? nullptr : c0, cz, o0, o1, oz, l, B, s,
                                   rot ? &rp : nullptr, in.rx, in.ry, in.mac);
    mark(5);
    return e;
}

// shared body of the key-switching calls: B ciphertexts whose c0 / c1 /
// outputs sit at stride `cz` words.
static int keyswitch_core(pc_ctx *c, const u32 *c0, const u32 *c1, size_t cz, u32 l, const pc_ksk *keys,
                          u32 B, u32 *o0, u32 *o1, cudaStream_t s, const KsInput &in = KsInput{},
                          bool profile = true) {
    const bool regen = keys[0].a == nullptr;
    for (u32 b = 1; b < B; ++b)
        if ((keys[b].a == nullptr) != regen) return PC_E_ARG;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (profile && cudaStreamIsCapturing(s, &cap) != cudaSuccess) cap = cudaStreamCaptureStatusNone;
    cudaEvent_t *ev = profile && cap == cudaStreamCaptureStatusNone ? profile_slot(c) : nullptr;
    // input checks (PC_CHECK_INPUTS): the ciphertext halves, the second
    // factor of a product, and the keys
    cudaError_t e = check_keys(c, keys, B, s);
    if (e == cudaSuccess && in.rx) e = check_ct(c, in.rx, 2 * l, l, 1, 0, s);
    if (e == cudaSuccess && in.ry) e = check_ct(c, in.ry, 2 * l, l, 1, 0, s);
    if (e == cudaSuccess && !in.rx) e = check_ct(c, c1, l, l, B, cz, s);
    if (e == cudaSuccess && c0) e = check_ct(c, c0, l, l, B, cz, s);
    if (e == cudaSuccess) e = ks_modup(c, c1, cz, l, B, B, in, s, ev);
    if (e == cudaSuccess) e = ks_finish(c, c0, c1, cz, l, keys, B, B, o0, o1, cz, in, s, ev);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

// do [a, a + an) and [b, b + bn) intersect
static bool overlaps(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + bn && y < x + an;
}

int pc_keyswitch(pc_ctx *c, const uint32_t *c0, const uint32_t *c1, uint32_t l, const pc_ksk *k,
                 uint32_t *c0o, uint32_t *c1o, pc_stream stream) {
    if (!c || !c0 || !c1 || !c0o || !c1o || l < 1 || l > c->L) return PC_E_ARG;
    if (int r = check_ksk(c, k)) return r;
    if (!aligned16(c0) || !aligned16(c1) || !aligned16(c0o) || !aligned16(c1o)) return PC_E_ALIGN;
    if (int r = need_ws(c, l, 1)) return r;
    DeviceGuard dg(c->device);
    return keyswitch_core(c, c0, c1, 0, l, k, 1, c0o, c1o, (cudaStream_t)stream);
}

// An executable graph of one key switch (fixed buffers, workspace and key).
struct pc_graph {
    pc_ctx *ctx;
    cudaGraph_t graph;
    cudaGraphExec_t exec;
};

int pc_capture_begin(pc_ctx *c, pc_stream *capture_stream) {
    if (!c || !capture_stream || c->cap) return PC_E_ARG;
    DeviceGuard dg(c->device);
    cudaStream_t cs = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) {
        if (cs) cudaStreamDestroy(cs);
        return cuda_fail(e);
    }
    c->cap = cs;
    *capture_stream = (pc_stream)cs;
    return PC_OK;
}

int pc_capture_end(pc_ctx *c, pc_graph **out) {
    if (out) *out = nullptr;
    if (!c || !c->cap) return PC_E_ARG;
    DeviceGuard dg(c->device);
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->cap, &g);
    cudaStreamDestroy(c->cap);
    c->cap = nullptr;
    if (e != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        return cuda_fail(e);
    }
    if (!out) {  // capture abandoned
        cudaGraphDestroy(g);
        return PC_OK;
    }
    cudaGraphExec_t x = nullptr;
    e = cudaGraphInstantiate(&x, g, 0);
    if (e != cudaSuccess) {
        cudaGraphDestroy(g);
        return cuda_fail(e);
    }
    *out = new (std::nothrow) pc_graph{c, g, x};
    if (!*out) {
        cudaGraphExecDestroy(x);
        cudaGraphDestroy(g);
        return PC_E_ARG;
    }
    return PC_OK;
}

int pc_keyswitch_capture(pc_ctx *c, const uint32_t *c0, const uint32_t *c1, uint32_t l, const pc_ksk *k,
                         uint32_t *c0o, uint32_t *c1o, pc_graph **out) {
    if (!out) return PC_E_ARG;
    *out = nullptr;
    if (!c || !c0 || !c1 || !c0o || !c1o || l < 1 || l > c->L) return PC_E_ARG;
    if (int r = check_ksk(c, k)) return r;
    if (!aligned16(c0) || !aligned16(c1) || !aligned16(c0o) || !aligned16(c1o)) return PC_E_ALIGN;
    if (int r = need_ws(c, l, 1)) return r;
    pc_stream cs = nullptr;
    if (int r = pc_capture_begin(c, &cs)) return r;
    const int rc = pc_keyswitch(c, c0, c1, l, k, c0o, c1o, cs);
    if (rc != PC_OK) {
        pc_capture_end(c, nullptr);
        return rc;
    }
    return pc_capture_end(c, out);
}

int pc_graph_launch(pc_graph *gr, pc_stream stream) {
    if (!gr) return PC_E_ARG;
    DeviceGuard dg(gr->ctx->device);
    const cudaError_t e = cudaGraphLaunch(gr->exec, (cudaStream_t)stream);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

void pc_graph_destroy(pc_graph *gr) {
    if (!gr) return;
    DeviceGuard dg(gr->ctx->device);
    cudaGraphExecDestroy(gr->exec);
    cudaGraphDestroy(gr->graph);
    delete gr;
}

int pc_keyswitch_batch(pc_ctx *c, const uint32_t *ct, uint32_t B, uint32_t l, const pc_ksk *keys,
                       uint32_t *out, pc_stream stream) {
    if (!c || !ct || !out || !keys || B < 1 || B > 64 || l < 1 || l > c->L) return PC_E_ARG;
    for (u32 b = 0; b < B; ++b)
        if (int r = check_ksk(c, &keys[b])) return r;
    if (!aligned16(ct) || !aligned16(out)) return PC_E_ALIGN;
    if (int r = need_ws(c, l, B)) return r;
    DeviceGuard dg(c->device);
    const size_t lN = (size_t)l * c->N;
    return keyswitch_core(c, ct, ct + lN, 2 * lN, l, keys, B, out, out + lN, (cudaStream_t)stream);
}

int pc_rotate(pc_ctx *c, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t galois, const pc_ksk *k,
              uint32_t *c0o, uint32_t *c1o, pc_stream stream) {
    if (!c || !c0 || !c1 || !c0o || !c1o || l < 1 || l > c->L || !galois_ok(c, galois)) return PC_E_ARG;
    if (int r = check_ksk(c, k)) return r;
    if (!aligned16(c0) || !aligned16(c1) || !aligned16(c0o) || !aligned16(c1o)) return PC_E_ALIGN;
    const size_t lb = (size_t)l * c->N * sizeof(u32);
    // the automorphism reads other rows than it writes: no in-place outputs
    if (overlaps(c0o, lb, c0, lb) || overlaps(c0o, lb, c1, lb) || overlaps(c1o, lb, c0, lb) ||
        overlaps(c1o, lb, c1, lb))
        return PC_E_ARG;
    if (int r = need_ws(c, l, 1)) return r;
    DeviceGuard dg(c->device);
    KsInput in;
    in.galois = galois;
    return keyswitch_core(c, c0, c1, 0, l, k, 1, c0o, c1o, (cudaStream_t)stream, in);
}

int pc_rotate_hoisted(pc_ctx *c, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t n,
                      const uint32_t *galois, const pc_ksk *keys, uint32_t *out, pc_stream stream) {
    if (!c || !c0 || !c1 || !out || !galois || !keys || l < 1 || l > c->L || n < 1 || n > 64) return PC_E_ARG;
    for (u32 i = 0; i < n; ++i) {
        if (!galois_ok(c, galois[i])) return PC_E_ARG;
        if (int r = check_ksk(c, &keys[i])) return r;
    }
    if (!aligned16(c0) || !aligned16(c1) || !aligned16(out)) return PC_E_ALIGN;
    const size_t lN = (size_t)l * c->N, ob = 2 * (size_t)n * lN * sizeof(u32);
    if (overlaps(out, ob, c0, lN * sizeof(u32)) || overlaps(out, ob, c1, lN * sizeof(u32))) return PC_E_ARG;
    // slices of up to KEYS_PER_LAUNCH rotations share one ModUp output
    const u32 Blay = n < (u32)pc::KEYS_PER_LAUNCH ? n : (u32)pc::KEYS_PER_LAUNCH;
    if (int r = need_ws(c, l, Blay)) return r;
    DeviceGuard dg(c->device);
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = check_keys(c, keys, n, s);
    if (e == cudaSuccess) e = check_ct(c, c0, l, l, 1, 0, s);
    if (e == cudaSuccess) e = check_ct(c, c1, l, l, 1, 0, s);
    if (e == cudaSuccess) e = ks_modup(c, c1, 0, l, 1, Blay, KsInput{}, s, nullptr);
    for (u32 i0 = 0; e == cudaSuccess && i0 < n; i0 += Blay) {
        const u32 nb = n - i0 < Blay ? n - i0 : Blay;
        KsInput in;
        in.hoist = galois + i0;
        u32 *o = out + 2 * (size_t)i0 * lN;
        e = ks_finish(c, c0, c1, 0, l, keys + i0, nb, Blay, o, o + lN, 2 * lN, in, s, nullptr);
    }
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_relinearize(pc_ctx *c, const uint32_t *x, const uint32_t *y, uint32_t l, const pc_ksk *k, uint32_t *out,
                   pc_stream stream) {
    if (!c || !x || !y || !out || l < 1 || l > c->L) return PC_E_ARG;
    if (int r = check_ksk(c, k)) return r;
    if (!aligned16(x) || !aligned16(y) || !aligned16(out)) return PC_E_ALIGN;
    const size_t lN = (size_t)l * c->N;
    const size_t cb = 2 * lN * sizeof(u32);
    if (overlaps(out, cb, x, cb) || overlaps(out, cb, y, cb)) return PC_E_ARG;
    if (int r = need_ws(c, l, 1)) return r;
    DeviceGuard dg(c->device);
    // key switch of d2 = x1 y1; d0 and d1 are formed in the final kernel
    KsInput in;
    in.mul = y + lN;
    in.rx = x;
    in.ry = y;
    return keyswitch_core(c, nullptr, x + lN, 0, l, k, 1, out, out + lN, (cudaStream_t)stream, in);
}

// pc_linear_transform: the key switch's workspace for the hoisted baby steps
// (up to 16 slices), then the n1 - 1 baby-step outputs [n1-1][2][l][N]
static u32 lt_slices(u32 n1) { return n1 <= 1 ? 1 : (n1 - 1 < (u32)pc::KEYS_PER_LAUNCH ? n1 - 1 : pc::KEYS_PER_LAUNCH); }
static size_t lt_ws_words(const pc_ctx *c, u32 l, u32 n1) {
    return layout(c, l, lt_slices(n1)).total + (size_t)(n1 - 1) * 2 * l * c->N;
}

size_t pc_linear_transform_workspace_bytes(const pc_ctx *c, uint32_t l, uint32_t n1) {
    if (!c || l < 1 || l > c->L || n1 < 1 || n1 > PC_BSGS_MAX_STEPS) return 0;
    return lt_ws_words(c, l, n1) * sizeof(u32);
}

int pc_linear_transform(pc_ctx *c, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t n1,
                        const uint32_t *g_baby, const pc_ksk *k_baby, uint32_t n2, const uint32_t *g_giant,
                        const pc_ksk *k_giant, const uint32_t *diag, uint32_t *out, pc_stream stream) {
    if (!c || !c0 || !c1 || !diag || !out || l < 1 || l > c->L) return PC_E_ARG;
    if (n1 < 1 || n2 < 1 || n1 > PC_BSGS_MAX_STEPS || n2 > PC_BSGS_MAX_STEPS) return PC_E_ARG;
    if ((n1 > 1 && (!g_baby || !k_baby)) || (n2 > 1 && (!g_giant || !k_giant))) return PC_E_ARG;
    for (u32 j = 0; j + 1 < n1; ++j) {
        if (!galois_ok(c, g_baby[j])) return PC_E_ARG;
        if (int r = check_ksk(c, &k_baby[j])) return r;
        if ((k_baby[j].a == nullptr) != (k_baby[0].a == nullptr)) return PC_E_ARG;  // one key mode per batch
    }
    for (u32 i = 0; i + 1 < n2; ++i) {
        if (!galois_ok(c, g_giant[i])) return PC_E_ARG;
        if (int r = check_ksk(c, &k_giant[i])) return r;
    }
    if (!aligned16(c0) || !aligned16(c1) || !aligned16(diag) || !aligned16(out)) return PC_E_ALIGN;
    const size_t lN = (size_t)l * c->N, b1 = lN * sizeof(u32);
    if (overlaps(out, 2 * b1, c0, b1) || overlaps(out, 2 * b1, c1, b1) ||
        overlaps(out, 2 * b1, diag, (size_t)n1 * n2 * b1))
        return PC_E_ARG;
    if (!c->ws || c->ws_bytes < lt_ws_words(c, l, n1) * sizeof(u32)) return PC_E_WORKSPACE;
    DeviceGuard dg(c->device);
    const cudaStream_t s = (cudaStream_t)stream;
    const u32 Blay = lt_slices(n1);
    u32 *bs = (u32 *)c->ws + layout(c, l, Blay).total;
    cudaError_t e = check_keys(c, k_baby, n1 - 1, s);
    if (e == cudaSuccess) e = check_keys(c, k_giant, n2 - 1, s);
    if (e == cudaSuccess) e = check_ct(c, c0, l, l, 1, 0, s);
    if (e == cudaSuccess) e = check_ct(c, c1, l, l, 1, 0, s);
    if (e == cudaSuccess) e = check_ct(c, diag, l, l, n1 * n2, lN, s);
    // baby steps: hoisted rotations of (c0, c1), one ModUp
    if (e == cudaSuccess && n1 > 1) e = ks_modup(c, c1, 0, l, 1, Blay, KsInput{}, s, nullptr);
    for (u32 j0 = 0; e == cudaSuccess && j0 + 1 < n1; j0 += Blay) {
        const u32 nb = n1 - 1 - j0 < Blay ? n1 - 1 - j0 : Blay;
        KsInput in;
        in.hoist = g_baby + j0;
        u32 *o = bs + 2 * (size_t)j0 * lN;
        e = ks_finish(c, c0, c1, 0, l, k_baby + j0, nb, Blay, o, o + lN, 2 * lN, in, s, nullptr);
    }
    // giant step 0: out = sum_j d_0j (.) bs_j; giant step i >= 1: out += the
    // rotation of W_i = sum_j d_ij (.) bs_j, W_i formed as the kernels read it
    pc::MacIn m{};
    m.x0[0] = c0;
    m.x0[1] = c1;
    m.xs = bs;
    m.xz = 2 * lN;
    m.hz = lN;
    m.d = diag;
    m.dz = lN;
    m.n1 = n1;
    if (e == cudaSuccess) e = pc::launch_mac(c, m, l, out, s);
    for (u32 i = 1; e == cudaSuccess && i < n2; ++i) {
        m.d = diag + (size_t)i * n1 * lN;
        KsInput in;
        in.galois = g_giant[i - 1];
        in.mac = &m;
        e = ks_modup(c, c1, 0, l, 1, 1, in, s, nullptr);
        if (e == cudaSuccess) e = ks_finish(c, c0, c1, 0, l, &k_giant[i - 1], 1, 1, out, out + lN, 0, in, s, nullptr);
    }
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_keyswitch_host(pc_ctx *c, const uint32_t *ct, uint32_t n, uint32_t l, const pc_ksk *keys, uint32_t *out,
                      pc_stream stream) {
    if (!c || !ct || !out || !keys || n < 1 || l < 1 || l > c->L) return PC_E_ARG;
    for (u32 k = 0; k < n; ++k)
        if (int r = check_ksk(c, &keys[k])) return r;
    const size_t lN = (size_t)l * c->N, cb = 2 * lN * sizeof(u32);
    if (overlaps(ct, n * cb, out, n * cb)) return PC_E_ARG;
    if (!c->ws || c->ws_bytes < host_ws_words(c, l) * sizeof(u32)) return PC_E_WORKSPACE;
    DeviceGuard dg(c->device);
    const cudaStream_t s = (cudaStream_t)stream;
    u32 *stage = (u32 *)c->ws + layout(c, l, 1).total;
    u32 *din[2] = {stage, stage + 4 * lN}, *dout[2] = {stage + 2 * lN, stage + 6 * lN};
    // the copy streams start after the work already queued on `stream`
    cudaError_t e = cudaEventRecord(c->ev_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->h2d, c->ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->d2h, c->ev_start, 0);
    int rc = e == cudaSuccess ? PC_OK : cuda_fail(e);
    for (u32 k = 0; rc == PC_OK && k < n; ++k) {
        const int i = k & 1;
        // slot i is free for input once key switch k-2 is done with it
        if (k >= 2) e = cudaStreamWaitEvent(c->h2d, c->ev_done[i], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(din[i], ct + k * 2 * lN, cb, cudaMemcpyHostToDevice, c->h2d);
        if (e == cudaSuccess) e = cudaEventRecord(c->ev_in[i], c->h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, c->ev_in[i], 0);
        // and free for output once copy k-2 has left it
        if (e == cudaSuccess && k >= 2) e = cudaStreamWaitEvent(s, c->ev_out[i], 0);
        if (e != cudaSuccess) { rc = cuda_fail(e); break; }
        rc = keyswitch_core(c, din[i], din[i] + lN, 0, l, &keys[k], 1, dout[i], dout[i] + lN, s);
        if (rc != PC_OK) break;
        e = cudaEventRecord(c->ev_done[i], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(c->d2h, c->ev_done[i], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(out + k * 2 * lN, dout[i], cb, cudaMemcpyDeviceToHost, c->d2h);
        if (e == cudaSuccess) e = cudaEventRecord(c->ev_out[i], c->d2h);
        if (e != cudaSuccess) rc = cuda_fail(e);
    }
    // `stream` completes only after every output has reached the host
    for (u32 k = n >= 2 ? n - 2 : 0; k < n; ++k) {
        const cudaError_t w = cudaStreamWaitEvent(s, c->ev_out[k & 1], 0);
        if (rc == PC_OK && w != cudaSuccess) rc = cuda_fail(w);
    }
    return rc;
}

int pc_expand_a(pc_ctx *c, const uint8_t seed[32], uint32_t l, uint32_t *a_out, pc_stream stream) {
    if (!c || !seed || !a_out || l < 1 || l > c->L) return PC_E_ARG;
    if (!aligned16(a_out)) return PC_E_ALIGN;
    DeviceGuard dg(c->device);
    u32 sw[8];
    seed_words(seed, sw);
    cudaError_t e = pc::launch_expand(c, sw, l, a_out, (cudaStream_t)stream);
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_profile_begin(pc_ctx *c, uint32_t max_calls, uint32_t every) {
    if (!c || max_calls < 1 || max_calls > 100000 || every < 1) return PC_E_ARG;
    DeviceGuard dg(c->device);
    prof_release(c);
    const size_t n = (size_t)max_calls * (PC_PROFILE_STAGES + 1);
    c->prof_ev = new (std::nothrow) cudaEvent_t[n];
    if (!c->prof_ev) return PC_E_ARG;
    for (size_t i = 0; i < n; ++i) {
        cudaError_t e = cudaEventCreate(&c->prof_ev[i]);
        if (e != cudaSuccess) {
            for (size_t k = 0; k < i; ++k) cudaEventDestroy(c->prof_ev[k]);
            delete[] c->prof_ev;
            c->prof_ev = nullptr;
            return cuda_fail(e);
        }
    }
    c->prof_max = max_calls;
    c->prof_used = 0;
    c->prof_every = every;
    c->prof_seen = 0;
    return PC_OK;
}

int pc_profile_end(pc_ctx *c, float *ms, uint32_t *calls) {
    if (!c || !ms) return PC_E_ARG;
    DeviceGuard dg(c->device);
    for (int k = 0; k < PC_PROFILE_STAGES; ++k) ms[k] = 0.f;
    if (calls) *calls = c->prof_used;
    int rc = PC_OK;
    for (uint32_t i = 0; i < c->prof_used && rc == PC_OK; ++i) {
        cudaEvent_t *ev = c->prof_ev + (size_t)i * (PC_PROFILE_STAGES + 1);
        cudaError_t e = cudaEventSynchronize(ev[PC_PROFILE_STAGES]);
        for (int k = 0; k < PC_PROFILE_STAGES && e == cudaSuccess; ++k) {
            float t = 0.f;
            e = cudaEventElapsedTime(&t, ev[k], ev[k + 1]);
            ms[k] += t;
        }
        if (e != cudaSuccess) rc = cuda_fail(e);
    }
    prof_release(c);
    return rc;
}

int pc_timeline_read(pc_ctx *c, uint64_t *out, size_t words) {
    if (!c || !out || words < (size_t)PC_TL_ROLES * PC_TL_CTAS * 3) return PC_E_ARG;
    DeviceGuard dg(c->device);
    const cudaError_t e = pc::timeline_read(c, out);
    if (e == cudaErrorNotSupported) return PC_E_UNSUPPORTED;
    return e == cudaSuccess ? PC_OK : cuda_fail(e);
}

int pc_check(pc_ctx *c) {
    if (!c) return PC_E_ARG;
    DeviceGuard dg(c->device);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    int word = 0;
    e = cudaMemcpy(&word, c->tab.err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (word) {
        c->last_err_word = (uint32_t)word;
        e = cudaMemset(c->tab.err, 0, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
        return PC_E_DEVICE;
    }
    return PC_OK;
}

uint32_t pc_last_error_word(const pc_ctx *c) { return c ? c->last_err_word : 0; }

int pc_set_checks(pc_ctx *c, uint32_t flags) {
    if (!c || (flags & ~(uint32_t)PC_CHECK_INPUTS)) return PC_E_ARG;
    c->checks = flags;
    return PC_OK;
}

const char *pc_strerror(int code) {
    switch (code) {
        case PC_OK: return "ok";
        case PC_E_ARG: return "invalid argument (null pointer, level or size out of range, bad parameters)";
        case PC_E_ALIGN: return "device pointer not 16-byte aligned (workspace: 256-byte)";
        case PC_E_CUDA: return cudaGetErrorString(g_last_cuda);
        case PC_E_DEVICE: return "an input check found a residue not below its prime (device error word set)";
        case PC_E_PRIME: return "modulus not prime, not 1 mod 2N, repeated, or >= 2^31";
        case PC_E_WORKSPACE: return "workspace missing or smaller than pc_workspace_bytes";
        case PC_E_TOO_BIG: return "l*N exceeds the static scratch of pc_modup_noalloc (2^21 words)";
        case PC_E_UNSUPPORTED: return "the library was built without the per-CTA timeline (build --timeline)";
        default: return "unknown status code";
    }
}

}  // extern "C"
