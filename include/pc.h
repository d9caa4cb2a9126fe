/*
 * pc.h -- C ABI of libpc: CKKS hybrid key switching over a 32-bit-word RNS
 * basis on one NVIDIA B200 (sm_100a), with the uniform 'a' half of every
 * key-switching key regenerated inside the kernel from a ChaCha12 seed.
 *
 * What the calls compute (the pages describe the operation, not its formula):
 *   - Perseus README (github gladia-research-group/perseus), "Layout": the
 *     device runtime provides the NTT and key switching over the 32-bit chain
 *     (intro: kernels descend from a 32-bit GPU port of FIDESlib);
 *   - same README, "What's inside": half of every key-switching key is
 *     regenerated on the GPU from a ChaCha12 seed instead of being stored;
 *   - "Perseus: A Full-Stack System for Homomorphic Model Inference"
 *     (arxivlens summary), "Methodology": a ChaCha12 counter-mode expander.
 * The formulas are the textbook ones (hybrid key switching of Han-Ki 2020;
 * full-RNS CKKS of Cheon-Han-Kim-Kim-Song 2018 with the approximate FastBConv
 * of Bajard-Eynard-Hasan-Zucca 2016), frozen as "spec v1" and stated at each
 * call below.
 *
 * Conventions for every call:
 *   - N = 2^logN, 10 <= logN <= 17.  Residues are uint32 in [0, q).
 *   - Global prime index g: 0..L-1 are the ciphertext primes q_g, L..L+alpha-1
 *     the special primes p_{g-L}.  At level l (1 <= l <= L, the number of q
 *     limbs) the local limb t in [0, l+alpha) is q_t for t < l and p_{t-l}
 *     otherwise.
 *   - Digit j at level l: D_j = {q_{j*alpha} .. q_{min(j*alpha+alpha, l)-1}},
 *     beta = ceil(l/alpha) digits (the last may be partial).
 *   - Polynomials are limb-major: [limb][N] uint32, in the NTT domain
 *     a_hat[k] = sum_n a[n] psi^((2 brv(k) + 1) n) mod q, psi the smallest
 *     primitive 2N-th root of unity mod q, brv the logN-bit reversal.
 *   - Pointers marked "device" are CUDA device pointers on the context's
 *     device, 16-byte aligned (else PC_E_ALIGN).  The caller owns every data
 *     buffer and the stream; no call allocates or frees device memory after
 *     pc_ctx_create.  Calls are asynchronous on `stream` (a cudaStream_t, 0 =
 *     legacy default stream); a return of PC_OK means "launched".
 *   - Buffers must not overlap unless a call says so.
 */
#ifndef PC_H
#define PC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define PC_OK 0
#define PC_E_ARG (-1)       /* null pointer, level/size out of range, bad params */
#define PC_E_ALIGN (-2)     /* a device pointer is not 16-byte aligned */
#define PC_E_CUDA (-3)      /* a CUDA call or launch failed (see pc_strerror) */
#define PC_E_DEVICE (-4)    /* an input check (pc_set_checks) set the device error word */
/* (-5) is not used: no call waits on the device with a time limit */
#define PC_E_PRIME (-6)     /* a modulus is not prime, not = 1 mod 2N, or >= 2^31 */
#define PC_E_WORKSPACE (-7) /* no workspace set, or smaller than pc_workspace_bytes */
#define PC_E_TOO_BIG (-8)   /* size beyond the static scratch of pc_modup_noalloc */
#define PC_E_UNSUPPORTED (-9) /* the call needs a library built with the per-CTA timeline */

typedef struct pc_ctx pc_ctx; /* opaque; owns the device constant tables */
typedef void *pc_stream;      /* a cudaStream_t */

/* RNS basis.  q: host array of L ciphertext primes; p: host array of alpha
 * special primes.  Every prime must be < 2^31 and = 1 mod 2N; all distinct.
 * dnum must equal ceil(L/alpha). */
typedef struct {
    uint32_t logN, L, alpha, dnum;
    const uint32_t *q;
    const uint32_t *p;
} pc_params;

/* A key-switching key for s' -> s ("packed": seed + stored 'b' half).
 *   seed: 32-byte ChaCha12 key of the 'a' half.
 *   b:    device, [dnum][L+alpha][N], NTT domain, indexed by global prime:
 *         b_{j,g} = -a_{j,g} s + e_j + [P]_{q_g} s' [q_g in D_j at the top level].
 *   a:    device or NULL.  NULL: a_{j,g} is regenerated in-kernel (spec v1
 *         mapping, see pc_expand_a).  Non-NULL: stored 'a' with b's layout. */
typedef struct {
    uint8_t seed[32];
    const uint32_t *b;
    const uint32_t *a;
} pc_ksk;

/* ---------------------------------------------------------------- */
/* parameters and context                                            */
/* ---------------------------------------------------------------- */

/* NTT-friendly primes below 2^bits (bits <= 31), host only: scan
 * k = floor((2^bits - 1)/2N) downward and keep c = k*2N + 1 when c is prime;
 * writes the first `count` found (largest first).  Spec v1 assigns the first
 * alpha of them to P and the next L to Q.  Returns PC_OK or PC_E_ARG. */
int pc_gen_primes(uint32_t logN, uint32_t bits, uint32_t count, uint32_t *out);

/* Validate the basis and build the device tables (twiddles, basis-conversion
 * constants) on `device`.  On success *out owns them; this is the only call
 * that allocates device memory.  Returns PC_OK, PC_E_ARG, PC_E_PRIME or
 * PC_E_CUDA. */
int pc_ctx_create(const pc_params *params, int device, pc_ctx **out);
void pc_ctx_destroy(pc_ctx *ctx);

/* psi (the smallest primitive 2N-th root) of global prime g, or 0 if g is out
 * of range.  Host only. */
uint32_t pc_psi(const pc_ctx *ctx, uint32_t g);

/* Bytes of device scratch that pc_keyswitch / pc_keyswitch_batch (B
 * ciphertexts), pc_modup and pc_moddown need at level l; and the call that
 * hands such a buffer (device, 256-byte aligned, owned by the caller, kept
 * until replaced) to the context.  Calls sharing one context and workspace
 * must be ordered on one stream. */
size_t pc_workspace_bytes(const pc_ctx *ctx, uint32_t l, uint32_t B);
int pc_set_workspace(pc_ctx *ctx, void *dev, size_t bytes);

/* ---------------------------------------------------------------- */
/* operations                                                        */
/* ---------------------------------------------------------------- */

/* Negacyclic NTT, in place.  x: device, [batch][nlimbs][N]; limb k of every
 * polynomial uses global prime first_prime + k (< L+alpha).  Forward maps
 * coefficients to the NTT domain defined above; inverse is its exact inverse
 * (N^-1 included).  Inputs in [0, q); outputs canonical. */
int pc_ntt_fwd(pc_ctx *ctx, uint32_t *x, uint32_t first_prime, uint32_t nlimbs,
               uint32_t batch, pc_stream stream);
int pc_ntt_inv(pc_ctx *ctx, uint32_t *x, uint32_t first_prime, uint32_t nlimbs,
               uint32_t batch, pc_stream stream);

/* ModUp (spec v1: approximate fast basis conversion per digit).
 * c1: device [l][N] NTT.  ext: device [beta][l+alpha][N] NTT, local limbs.
 * With x_i = INTT(c1_i): y_i = x_i [Dhat_i^-1]_{q_i}, Dhat_i = prod of the
 * digit's other primes; for t not in D_j, ext[j][t] = NTT_t(sum_i y_i [Dhat_i]_t
 * mod t); for t in D_j, ext[j][t] = c1[t].  Needs the workspace. */
int pc_modup(pc_ctx *ctx, const uint32_t *c1, uint32_t l, uint32_t *ext, pc_stream stream);

/* pc_modup without a workspace, for callers that cannot allocate device
 * memory (a plugin inside a host framework that owns every device allocation,
 * or a latency-critical path that cannot afford cudaMalloc's device-wide
 * synchronisation).  The pages have no counterpart of this call; it computes
 * exactly what pc_modup computes, with the same arguments and layouts, and
 * needs no pc_set_workspace.  Its l*N words of scratch live in one
 * statically allocated device array of 2^21 words (8 MiB) that the library
 * holds on every device it is loaded on until the process exits.  The
 * array's device address is looked up once per context, by pc_ctx_create,
 * with the context's device current (so this call does no lookup and may be
 * made at any time).  All calls share the array and it keeps the last call's
 * contents (nothing in it needs to start at zero); calls whose kernels overlap
 * on the GPU (two streams, or two host threads) race on it, so callers must
 * order them, e.g. on one stream.  Returns PC_OK, PC_E_ARG, PC_E_ALIGN,
 * PC_E_TOO_BIG (l*N above 2^21: N=2^16 up to l=32, N=2^17 up to l=16) or
 * PC_E_CUDA; never PC_E_WORKSPACE. */
int pc_modup_noalloc(pc_ctx *ctx, const uint32_t *c1, uint32_t l, uint32_t *ext, pc_stream stream);

/* Key inner product with in-kernel ChaCha12 regeneration of 'a'.
 * ext: device [beta][l+alpha][N] (pc_modup's output).  acc: device
 * [2][l+alpha][N]; acc[0][t] = sum_j ext[j][t] b_{j,g(t)} mod t (b half),
 * acc[1][t] = sum_j ext[j][t] a_{j,g(t)} mod t (a half).  a_{j,g} per
 * pc_expand_a when k->a is NULL.  No workspace. */
int pc_keyswitch_inner(pc_ctx *ctx, const uint32_t *ext, uint32_t l, const pc_ksk *k,
                       uint32_t *acc, pc_stream stream);

/* ModDown (spec v1: approximate conversion P -> Q_l, no rounding term).
 * acc: device [2][l+alpha][N] NTT.  out: device [2][l][N] NTT with, for each
 * half h, out[h][i] = (acc[h][i] - NTT(z_i)) [P^-1]_{q_i} where z_i =
 * sum_p [INTT(acc[h][p]) Phat_p^-1]_p [Phat_p]_{q_i} mod q_i; i.e.
 * floor(A/P) - v with v in [0, alpha).  Needs the workspace. */
int pc_moddown(pc_ctx *ctx, const uint32_t *acc, uint32_t l, uint32_t *out, pc_stream stream);

/* Full key switch s' -> s at level l: ModUp(c1), inner product, ModDown,
 * c0' = c0 + out[0], c1' = out[1].  c0, c1, c0o, c1o: device [l][N] NTT.
 * c0o may equal c0 and c1o may equal c1 (in place).  Needs the workspace. */
int pc_keyswitch(pc_ctx *ctx, const uint32_t *c0, const uint32_t *c1, uint32_t l,
                 const pc_ksk *k, uint32_t *c0o, uint32_t *c1o, pc_stream stream);

/* B independent key switches in one set of launches.  ct, out: device
 * [B][2][l][N] (c0 then c1 of each ciphertext); keys: host array of B keys
 * (ciphertext b uses keys[b]); out may equal ct.  1 <= B <= 64.  Needs the
 * workspace for B ciphertexts. */
int pc_keyswitch_batch(pc_ctx *ctx, const uint32_t *ct, uint32_t B, uint32_t l,
                       const pc_ksk *keys, uint32_t *out, pc_stream stream);

/* CUDA graph of one pc_keyswitch: pc_keyswitch_capture records the launches
 * of a key switch with these exact buffers, key and the context's current
 * workspace (including the internal stream's ModDown branch) into an
 * executable graph; pc_graph_launch replays it on `stream` (asynchronous),
 * computing exactly what pc_keyswitch computes, with one host call instead of
 * six launches and the fork/join events.  The buffers, the key's device
 * halves and the workspace must stay valid and unchanged in place while the
 * graph is used; calls sharing the context and workspace must still be
 * ordered on one stream.  Same arguments and status codes as pc_keyswitch
 * (out: the new graph, NULL on error).  The pages have no counterpart of
 * these calls. */
typedef struct pc_graph pc_graph;
int pc_keyswitch_capture(pc_ctx *ctx, const uint32_t *c0, const uint32_t *c1, uint32_t l, const pc_ksk *k,
                         uint32_t *c0o, uint32_t *c1o, pc_graph **out);

/* General capture: pc_capture_begin returns, in *capture_stream, a stream in
 * capture mode; the device-buffer calls (pc_keyswitch, pc_rotate,
 * pc_rotate_hoisted, pc_relinearize, pc_keyswitch_batch, the NTTs, ...) made
 * on it by this host thread are recorded, not run; pc_capture_end turns them
 * into an executable graph (*out; pass NULL to abandon the capture).  One
 * capture per context at a time (else PC_E_ARG).  Per-kernel profiling
 * events are not recorded in captured calls.  The same rules as for
 * pc_keyswitch_capture hold for the graph's buffers. */
int pc_capture_begin(pc_ctx *ctx, pc_stream *capture_stream);
int pc_capture_end(pc_ctx *ctx, pc_graph **out);
int pc_graph_launch(pc_graph *graph, pc_stream stream);
void pc_graph_destroy(pc_graph *graph);

/* Key switches of n ciphertexts held in HOST memory: ct and out are host
 * arrays [n][2][l][N] (c0 then c1 of each ciphertext, natural layout as in
 * device calls); keys: host array of n keys (device 'b' halves, as in
 * pc_keyswitch).  The library pipelines them through two device staging
 * slots: while ciphertext k is key-switched on `stream`, ciphertext k+1 is
 * copied in and ciphertext k-1 copied out on two internal streams, so copies
 * and kernels overlap (with page-locked host buffers; pageable ones work but
 * copy synchronously).  One cudaMemcpyAsync per ciphertext and direction.
 * Asynchronous: `stream` completes after the last output has reached the
 * host.  out must not overlap ct.  Needs a workspace of
 * pc_host_workspace_bytes(l) (the key switch's plus the staging slots), else
 * PC_E_WORKSPACE.  The pages have no counterpart of this call: it is the
 * host-facing entry point of the same key switch. */
size_t pc_host_workspace_bytes(const pc_ctx *ctx, uint32_t l);
int pc_keyswitch_host(pc_ctx *ctx, const uint32_t *ct, uint32_t n, uint32_t l, const pc_ksk *keys,
                      uint32_t *out, pc_stream stream);

/* Rotation: the key switch of c(X^g) = (c0(X^g), c1(X^g)) -- the ciphertext
 * under the automorphism X -> X^g, which decrypts under s(X^g) -- with a key
 * k for s(X^g) -> s.  (Perseus README, "Python API": the session holds keys
 * for the rotations a model uses, e.g. steps 1, 2, 4, 8, and
 * fhe.rotate_and_sum rotates by them; the pages give no formula, so this is
 * the textbook CKKS rotation: automorphism, then key switch.)  galois = g,
 * odd and < 2N (5^r mod 2N rotates the slots by r; 2N-1 conjugates), else
 * PC_E_ARG.  In the NTT domain X -> X^g permutes the slots: slot k of
 * x(X^g) is slot k' of x with 2 brv(k') + 1 = g (2 brv(k) + 1) mod 2N; the
 * kernels apply it while reading c1 and c0 (no permuted copy is made).
 * c0, c1, c0o, c1o: device [l][N] NTT; the outputs must not overlap the
 * inputs (PC_E_ARG).  Needs the workspace for (l, 1). */
int pc_rotate(pc_ctx *ctx, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t galois,
              const pc_ksk *k, uint32_t *c0o, uint32_t *c1o, pc_stream stream);

/* Hoisted rotations of one ciphertext by n Galois elements (the rotations of
 * one fhe.rotate_and_sum-style step list): ModUp of c1 runs once; rotation i
 * applies X -> X^galois[i] to the extended limbs ext_j inside the inner product
 * (a permuted ModUp output is a valid lift of c1(X^g)), then ModDown and
 * c0(X^g) as in pc_rotate.  galois, keys: host arrays of n (1 <= n <= 64);
 * keys[i] switches s(X^galois[i]) -> s.  out: device [n][2][l][N], rotation i
 * at out + 2 i l N (c0' then c1'), not overlapping c0 or c1.  Results equal
 * the hoisted oracle bit for bit; they differ from pc_rotate's only in the
 * ModUp approximation term, and both decrypt within the same bound.  The
 * rotations run in batches of up to 16 (one set of launches per batch), so
 * the call needs the workspace for (l, min(n, 16)), else PC_E_WORKSPACE. */
int pc_rotate_hoisted(pc_ctx *ctx, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t n,
                      const uint32_t *galois, const pc_ksk *keys, uint32_t *out, pc_stream stream);

/* Relinearisation of a ciphertext product (Perseus README, "Python API":
 * fhe.square; the textbook CKKS multiplication): the tensor of x = (x0, x1)
 * and y = (y0, y1) is (d0, d1, d2) = (x0 y0, x0 y1 + x1 y0, x1 y1) slot-wise
 * mod q_i (d0 + d1 s + d2 s^2 decrypts to the product), and d2 is key-switched
 * with a key k for s^2 -> s: out = (d0 + ModDown_b, d1 + ModDown_a).  The
 * tensor terms are formed inside the kernels that read x and y.  x, y, out:
 * device [2][l][N] NTT; out must not overlap x or y (PC_E_ARG); x may equal
 * y (squaring).  Needs the workspace for (l, 1). */
int pc_relinearize(pc_ctx *ctx, const uint32_t *x, const uint32_t *y, uint32_t l, const pc_ksk *k,
                   uint32_t *out, pc_stream stream);

/* Baby-step giant-step linear transform with hoisted baby steps: the
 * homomorphic matrix-vector product by the diagonal method that makes up the
 * CoeffsToSlots and SlotsToCoeffs steps of CKKS bootstrapping.  (Perseus
 * README, intro: GPT-2 runs 416 bootstraps per token; "Runtime": the `bts`
 * bootstrap bench of pc-bench; the HEAT listing: bootstraps dominate the
 * latency.  The pages give no formula, so this is the textbook method:
 * Halevi-Shoup diagonals split into baby and giant steps, Han-Ki 2020,
 * Chen-Chillotti-Song 2019.)
 *   bs_0 = (c0, c1); bs_j = rotation of (c0, c1) by g_baby[j-1], 1 <= j < n1,
 *          hoisted (one ModUp of c1; as pc_rotate_hoisted)
 *   W_i  = sum_{j < n1} diag[i][j] (.) bs_j        (slot-wise mod q)
 *   out  = W_0 + sum_{1 <= i < n2} rotation of W_i by g_giant[i-1]  (as pc_rotate)
 * diag: device [n2][n1][l][N], NTT-domain plaintexts (the caller's
 * pre-rotated diagonals), canonical.  g_baby, k_baby: host arrays of n1 - 1
 * Galois elements and keys (k_baby[j-1] switches s(X^g_baby[j-1]) -> s; all
 * baby keys regenerate their 'a' halves or all store them, else PC_E_ARG);
 * g_giant, k_giant: host arrays of n2 - 1 (may be NULL when n1 or n2 is 1).
 * 1 <= n1, n2 <= PC_BSGS_MAX_STEPS.  c0, c1: device [l][N]; out: device
 * [2][l][N] (c0' then c1'), not overlapping c0, c1 or diag (PC_E_ARG).  W_i
 * is never stored: the kernels that read a giant step's input form it from
 * the baby steps and diagonals, and the last kernel of each giant step adds
 * its result to out.  Needs a workspace of
 * pc_linear_transform_workspace_bytes(l, n1), else PC_E_WORKSPACE. */
#define PC_BSGS_MAX_STEPS 64
size_t pc_linear_transform_workspace_bytes(const pc_ctx *ctx, uint32_t l, uint32_t n1);
int pc_linear_transform(pc_ctx *ctx, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t n1,
                        const uint32_t *g_baby, const pc_ksk *k_baby, uint32_t n2, const uint32_t *g_giant,
                        const pc_ksk *k_giant, const uint32_t *diag, uint32_t *out, pc_stream stream);

/* Test hook: write the regenerated 'a' words for level l.  a_out: device
 * [beta][l+alpha][N], a_out[j][t][k] = a_{j,g(t)}[k] where (spec v1) block
 * b = k/8 of ChaCha12 with state words (constants "expand 32-byte k", seed as
 * eight little-endian words, counter b, g, j, 0x61) gives out[16], and
 * a = (out[2(k%8)+1] * 2^32 + out[2(k%8)]) mod q_g. */
int pc_expand_a(pc_ctx *ctx, const uint8_t seed[32], uint32_t l, uint32_t *a_out,
                pc_stream stream);

/* Input checks.  With PC_CHECK_INPUTS set, every operation above first runs
 * a kernel over the residues it reads (ciphertext limbs, accumulators,
 * extended limbs, both halves of every key) and sets bits of the context's
 * device error word for residues not below their prime: PC_ERR_INPUT for a
 * data operand, PC_ERR_KEY for a key half.  The check reads only the buffers
 * the call reads anyway, never traps, and does not stop the call; pc_check
 * reports the result.  Off by default (it reads every input once more).
 * flags: 0 or PC_CHECK_INPUTS, else PC_E_ARG. */
#define PC_CHECK_INPUTS 1u
#define PC_ERR_INPUT 1u
#define PC_ERR_KEY 2u
int pc_set_checks(pc_ctx *ctx, uint32_t flags);

/* Synchronise the context's device and read its device error word; returns
 * PC_OK, PC_E_DEVICE (the word was set: it is cleared, and its value kept
 * for pc_last_error_word), or PC_E_CUDA. */
int pc_check(pc_ctx *ctx);
uint32_t pc_last_error_word(const pc_ctx *ctx);

/* Human-readable text for a status code (the last CUDA error for PC_E_CUDA). */
const char *pc_strerror(int code);

/* ---------------------------------------------------------------- */
/* measurement                                                       */
/* ---------------------------------------------------------------- */

/* Integer-throughput microbenchmark on `device`: runs `iters` rounds of
 * independent modular-multiply chains (kind 0: Shoup multiply by a constant,
 * the form the NTT and basis conversions use; kind 1: Montgomery multiply of
 * two variables; kind 2: ChaCha12 blocks; kind 3: 32-bit multiply-add; kind
 * 4: xor + add; kinds 5..8: ChaCha12 blocks with some rotations computed on
 * the multiply pipe; kind 9: ChaCha12, two interleaved blocks; kind 10:
 * ChaCha12 with the 16- and 8-bit rotations as byte permutes; kinds 11..15:
 * single instructions of the transforms and the cipher, to find the pipe each
 * one issues on -- the conditional subtraction min(x, x - q), a funnel-shift
 * rotation, a byte-permute rotation, a 64-bit addition, a compare-and-select
 * subtraction) over all SMs and writes the operations per second to
 * *ops_per_s (modmuls/s, ChaCha blocks/s, or instructions/s).
 * Synchronous.  Returns PC_OK, PC_E_ARG or PC_E_CUDA. */
int pc_microbench(int device, int kind, uint32_t iters, double *ops_per_s);

/* Per-kernel timing of pc_keyswitch / pc_keyswitch_batch, for measurement.
 * pc_profile_begin creates CUDA events (host call, not on the hot path) for up
 * to max_calls sampled key-switch calls: of the calls that follow, every
 * `every`-th one (the 1st, the every+1-th, ...) records one event before each
 * of its PC_PROFILE_STAGES kernels and one after the last, on its stream;
 * the others run uninstrumented.  pc_profile_end synchronises, writes into
 * ms[PC_PROFILE_STAGES] the summed milliseconds of each stage over the
 * sampled calls (stages: 0 inverse row pass of c1; 1 ModUp column kernel:
 * inverse column pass + scale, basis conversion, forward column pass;
 * 2 inner product with ChaCha12 regeneration, forward row pass of the
 * converted limbs and inverse row pass of the special limbs; 3 ModDown
 * column kernel; 4 ModDown finish: forward row pass, scale, add), sets *calls
 * to the number of sampled calls, and releases the events.  Returns PC_OK,
 * PC_E_ARG or PC_E_CUDA. */
#define PC_PROFILE_STAGES 5
int pc_profile_begin(pc_ctx *ctx, uint32_t max_calls, uint32_t every);
int pc_profile_end(pc_ctx *ctx, float *ms, uint32_t *calls);

/* Per-CTA timeline of the key-switching kernels, for measurement.  Only a
 * library built with it (python -m key_switching_b200.build --timeline, which
 * writes libpc_timeline.so) records it: there every CTA of the kernels below
 * stores, as it exits, its start and end time (the GPU's global nanosecond
 * timer) and its SM id into a device array of PC_TL_ROLES x PC_TL_CTAS
 * records, at [role][CTA index within its grid], so each record holds the
 * latest launch of that role.  pc_timeline_read synchronises the context's
 * device, copies the array to host memory `out` (PC_TL_ROLES * PC_TL_CTAS * 3
 * uint64 words: start ns, end ns, SM) and zeroes it.  Roles: the inverse row
 * pass of c1 (ModUp), the conversion kernels of ModUp and ModDown, the inner
 * products of the special-prime and of the ciphertext-prime limbs
 * (two-group kernel), the ModDown finish, other row passes, the single-group
 * and rotation inner products.  CTAs beyond PC_TL_CTAS are not recorded.
 * Returns PC_OK, PC_E_ARG (null or `words` too small), PC_E_UNSUPPORTED
 * (default build) or PC_E_CUDA. */
#define PC_TL_ROLES 8
#define PC_TL_CTAS 4096
#define PC_TL_ROW_C1 0
#define PC_TL_CONV_UP 1
#define PC_TL_INNER_SPECIAL 2
#define PC_TL_CONV_DOWN 3
#define PC_TL_INNER_CT 4
#define PC_TL_MODDOWN_FINISH 5
#define PC_TL_ROW_OTHER 6
#define PC_TL_INNER_OTHER 7
int pc_timeline_read(pc_ctx *ctx, uint64_t *out, size_t words);

#ifdef __cplusplus
}
#endif
#endif /* PC_H */
