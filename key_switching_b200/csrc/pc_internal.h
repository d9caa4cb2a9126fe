// pc_internal.h -- context, device tables and launchers shared by the
// libpc translation units (never exported).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/pc.h"

namespace pc {

typedef uint32_t u32;
typedef uint64_t u64;

constexpr int MAX_L = 64;       // ciphertext primes
constexpr int MAX_ALPHA = 8;    // special primes (digit size)
constexpr int KEYS_PER_LAUNCH = 16;

// Per-prime constants (device).  Shoup companions w' = floor(w 2^32 / q).
struct PrimeK {
    u32 q;
    u32 qn;          // -q^-1 mod 2^32 (REDC)
    u32 q1s;         // floor(2^32 / q)
    u32 r32, r32s;   // 2^32 mod q
    u32 r64, r64s;   // 2^64 mod q
    u32 ninv, ninvs; // N^-1 mod q
    u32 pad[7];
};

// Device tables of one context, passed to kernels by value.
struct Tables {
    const PrimeK *pk;        // [NP]
    const uint2 *colF;       // [NP][R]  psi_rev[k], k < R
    const uint2 *colI;       // [NP][R]  psi^-1 rev
    const uint2 *rowF;       // [NP][R][C] per-row re-laid twiddles
    const uint2 *rowI;       // [NP][R][C]
    const uint2 *upScale;    // [alpha][L]: N^-1 [Dhat_i^-1]_{q_i}, digit of size d at index d-1
    const u32 *upConv;       // [dnum][alpha][NP][alpha]: [Dhat_k mod g] 2^32 mod g
    const uint2 *downScale;  // [alpha]: N^-1 [Phat_k^-1]_{p_k}
    const u32 *downConv;     // [L][alpha]: [Phat_k mod q_i] 2^32 mod q_i
    const uint2 *pInv;       // [L]: [P^-1]_{q_i}
    int *err;                // device error word
    u32 L, alpha, dnum, NP;
};

// Up to KEYS_PER_LAUNCH keys, by value in the kernel parameters.
struct KeyPack {
    const u32 *b[KEYS_PER_LAUNCH];
    const u32 *a[KEYS_PER_LAUNCH];
    u32 seed[KEYS_PER_LAUNCH][8];
};

// Automorphism X -> X^galois[z] (and galois[z]^-1 mod 2N) for grid slice z
// of a rotation launch, by value in the kernel parameters; 1 = none.
struct RotPack {
    u32 galois[KEYS_PER_LAUNCH];
    u32 ginv[KEYS_PER_LAUNCH];
};

// Operand of a giant step of a baby-step giant-step linear transform: half h
// of W = sum_{j < n1} d_j (.) bs_j (slot-wise mod q), where bs_0 is the input
// ciphertext (half h at x0[h]), baby step j >= 1 has half h at
// xs + (j-1) xz + h hz, and diagonal j is at d + j dz; limb i of each at + i N.
struct MacIn {
    const u32 *x0[2];
    const u32 *xs;
    size_t xz, hz;
    const u32 *d;
    size_t dz;
    u32 n1;
};

}  // namespace pc

struct pc_ctx {
    int device;
    int num_sms;
    uint32_t logN, N, L, alpha, dnum, NP;
    uint32_t primes[pc::MAX_L + pc::MAX_ALPHA];
    uint32_t psi[pc::MAX_L + pc::MAX_ALPHA];
    pc::Tables tab;
    void *dev_block;  // one allocation holding every table
    size_t dev_bytes;
    void *ws;         // caller's workspace
    size_t ws_bytes;
    // device address of the static scratch array of pc_modup_noalloc on
    // this context's device (looked up at context creation)
    uint32_t *noalloc_scratch;
    // PC_CHECK_* flags of pc_set_checks: validate inputs on the device
    uint32_t checks;
    uint32_t last_err_word;  // the error word pc_check last found set
    // CTAs of the conversion kernel resident at once on the device (0: never
    // split its items by target; PC_COLCONV_SPLIT=0)
    uint32_t colconv_slots;
    // launch attributes: programmatic dependent launch, L2 persistence of the tables
    int use_pdl;
    void *l2_window_base;
    size_t l2_window_bytes;
    float l2_hit_ratio;
    // internal high-priority stream and fork / join events: the ModDown
    // branch of a key switch overlaps the ciphertext-prime inner products
    int overlap;
    cudaStream_t aux;
    cudaEvent_t ev_fork, ev_join;
    // host-buffer pipeline (pc_keyswitch_host): copy streams and, per staging
    // slot, "input landed", "key switch done" and "output copied" events
    cudaStream_t h2d, d2h;
    cudaEvent_t ev_start, ev_in[2], ev_done[2], ev_out[2];
    // stream in capture mode between pc_capture_begin and pc_capture_end
    cudaStream_t cap;
    // per-kernel timing (pc_profile_begin / pc_profile_end)
    cudaEvent_t *prof_ev;   // [prof_max][PC_PROFILE_STAGES + 1]
    uint32_t prof_max, prof_used, prof_every, prof_seen;
};

namespace pc {

// launchers (kernels.cu); each returns a cudaError_t from the launch.
// "CM" = column-major limb (element (r, c) at c*R + r), used for the
// intermediates between row passes and column passes.
// The inverse pass can read its input limbs through X -> X^galois and / or
// times the limbs of `mul` (same strides), and store that transformed input
// (row-major, stride zout) to xout.
// With mac (inverse, Z = 1): the input limbs are half 1 of the giant-step
// operand W of *mac (see MacIn) instead of `in`, read through X -> X^galois.
cudaError_t launch_row(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, bool canonical, bool cm_out, cudaStream_t s, u32 galois = 1,
                       const u32 *mul = nullptr, u32 *xout = nullptr, const MacIn *mac = nullptr);
// scale_mode: 0 none (lazy), 1 N^-1 (canonical)
cudaError_t launch_col(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, int scale_mode, cudaStream_t s);
// conversion kernel: inverse column pass + scale of the sources (CM), basis
// conversion and forward column pass of the targets.  mode 0 (ModUp):
// src = INTT-row output of c1 (CM) [l][N], out = [beta][l+alpha][N];
// mode 1 (ModDown): src = ACC [2][l+alpha][N] (special limbs CM),
// out = [2][l][N].  Output CM when out_cm, else row-major.
cudaError_t launch_colconv(const pc_ctx *c, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz, u32 l,
                           u32 Z, bool out_cm, cudaStream_t s);
// inner product for target limbs t0 .. t0+nt-1 (nt = 0: through l+alpha-1).
// rot (fused only) applies X -> X^galois[z] to the extended limbs of slice z
// (hoisted rotations).
cudaError_t launch_inner(const pc_ctx *c, bool fused, const u32 *src, size_t srcz, const u32 *c1, size_t c1z,
                         u32 *acc, size_t accz, u32 l, const KeyPack &kp, u32 Z, bool regen, bool pintt,
                         cudaStream_t s, u32 t0 = 0, u32 nt = 0, const RotPack *rot = nullptr);
// ModDown finish; c0 of slice z read through X -> X^galois[z] when rot is
// given, or (rx, ry given) the tensor terms d0, d1 of ciphertexts rx, ry
// added instead of c0, or (mac given, Z = 1) half 0 of the giant-step operand
// W of *mac read through X -> X^galois[0] instead of c0, and the result added
// to the outputs' previous contents.
cudaError_t launch_moddown_row(const pc_ctx *c, const u32 *U, size_t Uz, const u32 *acc, size_t accz, const u32 *c0,
                               size_t c0z, u32 *out0, u32 *out1, size_t outz, u32 l, u32 Z, cudaStream_t s,
                               const RotPack *rot = nullptr, const u32 *rx = nullptr, const u32 *ry = nullptr,
                               const MacIn *mac = nullptr);
// out[h][i] = sum_j d_j (.) bs_j half h (the giant step without rotation),
// out: [2][l][N] canonical.
cudaError_t launch_mac(const pc_ctx *c, const MacIn &m, u32 l, u32 *out, cudaStream_t s);
cudaError_t launch_modup_finish(const pc_ctx *c, const u32 *c1, u32 *ext, u32 l, cudaStream_t s);
cudaError_t launch_expand(const pc_ctx *c, const u32 seed[8], u32 l, u32 *out, cudaStream_t s);
// Input validation: OR `bit` into the device error word if any residue of
// x is not below its prime.  x holds Z slices (stride zs words) of nlimbs
// limbs of N words; limb t uses prime: mode 0, global index first + t;
// mode 1, the local limb (t mod period) at level l; mode 2, the global index
// t mod period (a key half [dnum][L+alpha][N]).
cudaError_t launch_check(const pc_ctx *c, const u32 *x, u32 nlimbs, u32 Z, size_t zs, int mode, u32 first,
                         u32 period, u32 l, int bit, cudaStream_t s);
// Look up the device address of pc_modup_noalloc's static scratch array on
// the context's device (which must be current) into c->noalloc_scratch.
cudaError_t noalloc_setup(pc_ctx *c);

// Make `dev` the current device for the lifetime of the guard, then restore
// the caller's device.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
    DeviceGuard(const DeviceGuard &) = delete;
    DeviceGuard &operator=(const DeviceGuard &) = delete;
};
// Per-degree set-up: shared-memory limits of the kernels and the number of
// conversion-kernel CTAs resident on the device (colconv_slots)
cudaError_t prepare_kernels(pc_ctx *c);
// copy out and zero the per-CTA timeline of the context's degree
// (cudaErrorNotSupported unless built with PC_TIMELINE)
cudaError_t timeline_read(const pc_ctx *c, uint64_t *out);

// Remember a CUDA error for pc_strerror(PC_E_CUDA); returns PC_E_CUDA.
int record_cuda_error(cudaError_t e);

}  // namespace pc
