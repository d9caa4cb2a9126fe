/*
 * oracle.c -- plain, slow CPU reference for CKKS hybrid key switching with a
 * ChaCha12-regenerated uniform key half.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this code.  The CUDA library never calls
 * it, links it or shares a header, table or helper with it.
 *
 * What it computes, and where it comes from:
 *   - Perseus README (github gladia-research-group/perseus), "What's inside":
 *     half of every key-switching key is regenerated on the GPU from a ChaCha12
 *     seed instead of being stored; "Layout": the device runtime does NTT and
 *     key switching over a 32-bit RNS chain (FIDESlib32bits descent, intro).
 *   - "Perseus: A Full-Stack System for Homomorphic Model Inference" (arxivlens
 *     summary), "Methodology": in-kernel regeneration of key-switching keys
 *     with a ChaCha12 counter-mode expander, halving key storage.
 * The pages give no formula for any step, so every step below is the plain
 * textbook reading, frozen as "spec v1":
 *   - hybrid key switching: Han & Ki, "Better bootstrapping for approximate
 *     HE" (CT-RSA 2020), digits of alpha consecutive primes;
 *   - full-RNS CKKS basis conversion: Cheon, Han, Kim, Kim, Song (SAC 2018),
 *     approximate FastBConv of Bajard, Eynard, Hasan, Zucca (SAC 2016);
 *   - negacyclic NTT: Longa & Naehrig (CANS 2016), merged psi powers,
 *     bit-reversed output order;
 *   - ChaCha: Bernstein (2008), 12 rounds, counter mode.
 * Every multiply is a 64-bit product reduced with '%'; nothing is lazy.
 *
 * Parity: pinned by tests/test_oracle_*.py against closed forms, brute force
 * at tiny sizes, Python big-integer CRT, the `cryptography` package's ChaCha20,
 * and decryption after key switching under the true secret.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* modular helpers (plain '%')                                         */
/* ------------------------------------------------------------------ */

static uint32_t mulm(uint32_t a, uint32_t b, uint32_t q) {
    return (uint32_t)(((uint64_t)a * (uint64_t)b) % q);
}
static uint32_t addm(uint32_t a, uint32_t b, uint32_t q) {
    return (uint32_t)(((uint64_t)a + (uint64_t)b) % q);
}
static uint32_t subm(uint32_t a, uint32_t b, uint32_t q) {
    return (uint32_t)(((uint64_t)a + (uint64_t)q - (uint64_t)b) % q);
}
static uint32_t powm(uint32_t a, uint64_t e, uint32_t q) {
    uint64_t r = 1 % q, x = a % q;
    while (e) {
        if (e & 1) r = (r * x) % q;
        x = (x * x) % q;
        e >>= 1;
    }
    return (uint32_t)r;
}
/* inverse by Fermat (q prime) */
static uint32_t invm(uint32_t a, uint32_t q) { return powm(a, (uint64_t)q - 2, q); }

static uint32_t bitrev(uint32_t x, uint32_t bits) {
    uint32_t r = 0;
    for (uint32_t i = 0; i < bits; i++) r |= ((x >> i) & 1u) << (bits - 1 - i);
    return r;
}

/* ------------------------------------------------------------------ */
/* primes and roots                                                    */
/* ------------------------------------------------------------------ */

/* Deterministic Miller-Rabin for n < 2^32 with witnesses 2, 7, 61
 * (Jaeschke 1993: these three witnesses decide every n < 4,759,123,141). */
int or_is_prime(uint32_t n) {
    static const uint32_t wit[3] = {2, 7, 61};
    if (n < 2) return 0;
    if (n % 2 == 0) return n == 2;
    uint32_t d = n - 1, s = 0;
    while ((d & 1) == 0) { d >>= 1; s++; }
    for (int k = 0; k < 3; k++) {
        uint32_t a = wit[k] % n;
        if (a == 0) continue;
        uint32_t x = powm(a, d, n);
        if (x == 1 || x == n - 1) continue;
        int comp = 1;
        for (uint32_t r = 1; r < s; r++) {
            x = mulm(x, x, n);
            if (x == n - 1) { comp = 0; break; }
        }
        if (comp) return 0;
    }
    return 1;
}

/* NTT-friendly primes below 2^bits: scan k downward from floor((2^bits-1)/2N)
 * and keep c = k*2N + 1 when c is prime; the first `count` found, in order
 * (largest first).  Returns 0, or -1 if the scan runs out. */
int or_gen_primes(uint32_t logN, uint32_t bits, uint32_t count, uint32_t *out) {
    uint64_t twoN = 2ull << logN;
    uint64_t k = (((uint64_t)1 << bits) - 1) / twoN;
    uint32_t found = 0;
    while (found < count) {
        if (k == 0) return -1;
        uint64_t c = k * twoN + 1;
        if (c < ((uint64_t)1 << 32) && or_is_prime((uint32_t)c)) out[found++] = (uint32_t)c;
        k--;
    }
    return 0;
}

/* The smallest x >= 2 with x^N = -1 mod q: the smallest primitive 2N-th root
 * of unity (x^N = -1 forces order exactly 2N). */
static uint32_t min_psi_search(uint32_t q, uint32_t logN) {
    uint64_t N = 1ull << logN;
    for (uint32_t x = 2; x < q; x++)
        if (powm(x, N, q) == q - 1) return x;
    return 0;
}

/* memo of the search above (the search is the definition; the memo only
 * avoids repeating it for every limb) */
uint32_t or_min_psi(uint32_t q, uint32_t logN) {
    enum { SLOTS = 512 };
    static uint32_t mq[SLOTS], ml[SLOTS], mv[SLOTS];
    static int used = 0;
    for (int i = 0; i < used; i++)
        if (mq[i] == q && ml[i] == logN) return mv[i];
    uint32_t v = min_psi_search(q, logN);
    if (used < SLOTS) { mq[used] = q; ml[used] = logN; mv[used] = v; used++; }
    return v;
}

/* ------------------------------------------------------------------ */
/* negacyclic NTT                                                      */
/* ------------------------------------------------------------------ */
/* Definition (spec v1): a_hat[k] = sum_n a[n] * psi^((2*brv(k)+1)*n) mod q,
 * brv over logN bits.  Computed by the in-place Cooley-Tukey butterfly
 * network with psi^brv(m+i) twiddles (Longa-Naehrig), which yields exactly
 * that bit-reversed evaluation order.  The inverse is the Gentleman-Sande
 * network with inverse twiddles followed by multiplication by N^-1. */

void or_ntt_fwd(uint32_t *a, uint32_t logN, uint32_t q, uint32_t psi) {
    uint32_t N = 1u << logN;
    uint32_t *tw = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (uint32_t k = 0; k < N; k++) tw[k] = powm(psi, bitrev(k, logN), q);
    uint32_t t = N;
    for (uint32_t m = 1; m < N; m <<= 1) {
        t >>= 1;
        for (uint32_t i = 0; i < m; i++) {
            uint32_t w = tw[m + i];
            uint32_t j1 = 2 * i * t;
            for (uint32_t j = j1; j < j1 + t; j++) {
                uint32_t u = a[j], v = mulm(a[j + t], w, q);
                a[j] = addm(u, v, q);
                a[j + t] = subm(u, v, q);
            }
        }
    }
    free(tw);
}

void or_ntt_inv(uint32_t *a, uint32_t logN, uint32_t q, uint32_t psi) {
    uint32_t N = 1u << logN;
    uint32_t psi_inv = invm(psi, q);
    uint32_t *tw = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (uint32_t k = 0; k < N; k++) tw[k] = powm(psi_inv, bitrev(k, logN), q);
    uint32_t t = 1;
    for (uint32_t m = N >> 1; m >= 1; m >>= 1) {
        for (uint32_t i = 0; i < m; i++) {
            uint32_t w = tw[m + i];
            uint32_t j1 = 2 * i * t;
            for (uint32_t j = j1; j < j1 + t; j++) {
                uint32_t u = a[j], v = a[j + t];
                a[j] = addm(u, v, q);
                a[j + t] = mulm(subm(u, v, q), w, q);
            }
        }
        t <<= 1;
    }
    uint32_t ninv = invm(N % q, q);
    for (uint32_t j = 0; j < N; j++) a[j] = mulm(a[j], ninv, q);
    free(tw);
}

/* ------------------------------------------------------------------ */
/* ChaCha                                                              */
/* ------------------------------------------------------------------ */
/* Bernstein's ChaCha: 16-word state, quarter-round with rotations
 * 16, 12, 8, 7; a double round is four column quarter-rounds followed by
 * four diagonal ones; the block is the permuted state plus the input state,
 * word-wise mod 2^32. */

static uint32_t rotl(uint32_t x, int r) { return (x << r) | (x >> (32 - r)); }

static void qround(uint32_t *x, int a, int b, int c, int d) {
    x[a] += x[b]; x[d] ^= x[a]; x[d] = rotl(x[d], 16);
    x[c] += x[d]; x[b] ^= x[c]; x[b] = rotl(x[b], 12);
    x[a] += x[b]; x[d] ^= x[a]; x[d] = rotl(x[d], 8);
    x[c] += x[d]; x[b] ^= x[c]; x[b] = rotl(x[b], 7);
}

/* the permutation alone, `double_rounds` double rounds, no feed-forward */
void or_chacha_permute(uint32_t x[16], int double_rounds) {
    for (int i = 0; i < double_rounds; i++) {
        qround(x, 0, 4, 8, 12);
        qround(x, 1, 5, 9, 13);
        qround(x, 2, 6, 10, 14);
        qround(x, 3, 7, 11, 15);
        qround(x, 0, 5, 10, 15);
        qround(x, 1, 6, 11, 12);
        qround(x, 2, 7, 8, 13);
        qround(x, 3, 4, 9, 14);
    }
}

/* ChaCha block with `rounds` rounds (12 for the method; 20 only for pins) */
void or_chacha_block(const uint32_t in[16], int rounds, uint32_t out[16]) {
    uint32_t x[16];
    memcpy(x, in, sizeof(x));
    or_chacha_permute(x, rounds / 2);
    for (int i = 0; i < 16; i++) out[i] = x[i] + in[i];
}

/* Spec v1 word layout of the key-regeneration stream for digit j and global
 * prime index g: constants "expand 32-byte k", the 32-byte seed as eight
 * little-endian words, the block counter, g, j, and the tag 0x61 ('a'). */
static void chacha_state(uint32_t st[16], const uint8_t seed[32], uint32_t ctr,
                         uint32_t g, uint32_t j) {
    st[0] = 0x61707865u; st[1] = 0x3320646eu; st[2] = 0x79622d32u; st[3] = 0x6b206574u;
    for (int w = 0; w < 8; w++)
        st[4 + w] = (uint32_t)seed[4 * w] | ((uint32_t)seed[4 * w + 1] << 8) |
                    ((uint32_t)seed[4 * w + 2] << 16) | ((uint32_t)seed[4 * w + 3] << 24);
    st[12] = ctr; st[13] = g; st[14] = j; st[15] = 0x61u;
}

/* a_{j,g}[k] for k < N (NTT domain): block b = k/8, words lo = out[2(k%8)],
 * hi = out[2(k%8)+1], a = (hi*2^32 + lo) mod q. */
void or_expand_a(const uint8_t seed[32], uint32_t j, uint32_t g, uint32_t q,
                 uint32_t logN, int rounds, uint32_t *out) {
    uint32_t N = 1u << logN;
    uint32_t st[16], ks[16];
    for (uint32_t b = 0; b < N / 8; b++) {
        chacha_state(st, seed, b, g, j);
        or_chacha_block(st, rounds, ks);
        for (uint32_t w = 0; w < 8; w++) {
            uint64_t v = ((uint64_t)ks[2 * w + 1] << 32) | (uint64_t)ks[2 * w];
            out[8 * b + w] = (uint32_t)(v % q);
        }
    }
}

/* ------------------------------------------------------------------ */
/* parameters                                                          */
/* ------------------------------------------------------------------ */

typedef struct {
    uint32_t logN, L, alpha, dnum;
    const uint32_t *q; /* L ciphertext primes */
    const uint32_t *p; /* alpha special primes */
} or_params;

static uint32_t prime_of(const or_params *P, uint32_t g) {
    return g < P->L ? P->q[g] : P->p[g - P->L];
}
/* local limb t at level l -> global prime index */
static uint32_t glob(const or_params *P, uint32_t l, uint32_t t) {
    return t < l ? t : P->L + (t - l);
}
static int check_params(const or_params *P, uint32_t l) {
    if (!P || !P->q || !P->p || P->alpha == 0 || P->L == 0) return -1;
    if (P->dnum != (P->L + P->alpha - 1) / P->alpha) return -1;
    if (l < 1 || l > P->L) return -1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* ModUp: approximate fast basis conversion per digit                  */
/* ------------------------------------------------------------------ */
/* Digit D_j = {q_{j*alpha}, ..., q_{min(j*alpha+alpha, l)-1}}, beta = ceil(l/alpha).
 * With x_i the coefficient form of c1 mod q_i:
 *   y_i = x_i * [Dhat_i^-1]_{q_i} mod q_i,  Dhat_i = prod_{k in D_j, k != i} q_k,
 *   z_t = (sum_i y_i * [Dhat_i]_t) mod t   for every t in (Q_l u P) \ D_j,
 * then ext_j[t] = NTT_t(z_t); the digit's own limbs are the input limbs.
 * c1: [l][N] NTT domain; ext: [beta][l+alpha][N] NTT domain, local indexing. */
int or_modup(const or_params *P, const uint32_t *c1, uint32_t l, uint32_t *ext) {
    if (check_params(P, l)) return -1;
    uint32_t N = 1u << P->logN, a = P->alpha, beta = (l + a - 1) / a, ll = l + a;
    uint32_t *x = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)l * N);
    uint32_t *z = (uint32_t *)malloc(sizeof(uint32_t) * N);
    /* coefficient form of every limb of c1 */
    for (uint32_t i = 0; i < l; i++) {
        uint32_t q = P->q[i];
        memcpy(x + (size_t)i * N, c1 + (size_t)i * N, sizeof(uint32_t) * N);
        or_ntt_inv(x + (size_t)i * N, P->logN, q, or_min_psi(q, P->logN));
    }
    for (uint32_t j = 0; j < beta; j++) {
        uint32_t lo = j * a, hi = (j * a + a < l) ? j * a + a : l;
        uint32_t *y = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(hi - lo) * N);
        for (uint32_t i = lo; i < hi; i++) {
            uint32_t qi = P->q[i], dh = 1;
            for (uint32_t k = lo; k < hi; k++)
                if (k != i) dh = mulm(dh, P->q[k] % qi, qi);
            uint32_t dinv = invm(dh, qi);
            for (uint32_t n = 0; n < N; n++)
                y[(size_t)(i - lo) * N + n] = mulm(x[(size_t)i * N + n], dinv, qi);
        }
        for (uint32_t t = 0; t < ll; t++) {
            uint32_t *dst = ext + ((size_t)j * ll + t) * N;
            if (t >= lo && t < hi) {
                memcpy(dst, c1 + (size_t)t * N, sizeof(uint32_t) * N);
                continue;
            }
            uint32_t mt = prime_of(P, glob(P, l, t));
            for (uint32_t n = 0; n < N; n++) z[n] = 0;
            for (uint32_t i = lo; i < hi; i++) {
                uint32_t dh = 1; /* Dhat_i mod t */
                for (uint32_t k = lo; k < hi; k++)
                    if (k != i) dh = mulm(dh, P->q[k] % mt, mt);
                for (uint32_t n = 0; n < N; n++)
                    z[n] = addm(z[n], mulm(y[(size_t)(i - lo) * N + n] % mt, dh, mt), mt);
            }
            memcpy(dst, z, sizeof(uint32_t) * N);
            or_ntt_fwd(dst, P->logN, mt, or_min_psi(mt, P->logN));
        }
        free(y);
    }
    free(z);
    free(x);
    return 0;
}

/* ------------------------------------------------------------------ */
/* key inner product                                                   */
/* ------------------------------------------------------------------ */
/* acc_b[t] = sum_{j<beta} ext_j[t] * b_{j,g(t)}   mod t
 * acc_a[t] = sum_{j<beta} ext_j[t] * a_{j,g(t)}   mod t
 * b: [dnum][L+alpha][N] NTT domain, read at global prime index g(t);
 * a: NULL -> regenerated from the seed by ChaCha (rounds), else stored with
 *    b's layout.  acc: [2][l+alpha][N], half 0 = b-half, half 1 = a-half. */
int or_inner(const or_params *P, const uint32_t *ext, uint32_t l, const uint8_t seed[32],
             const uint32_t *b, const uint32_t *a, int rounds, uint32_t *acc) {
    if (check_params(P, l) || !b) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, beta = (l + al - 1) / al, ll = l + al;
    uint32_t LL = P->L + al;
    uint32_t *ak = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (uint32_t t = 0; t < ll; t++) {
        uint32_t g = glob(P, l, t), mt = prime_of(P, g);
        uint32_t *ob = acc + (size_t)t * N, *oa = acc + ((size_t)ll + t) * N;
        for (uint32_t n = 0; n < N; n++) { ob[n] = 0; oa[n] = 0; }
        for (uint32_t j = 0; j < beta; j++) {
            const uint32_t *e = ext + ((size_t)j * ll + t) * N;
            const uint32_t *bj = b + ((size_t)j * LL + g) * N;
            const uint32_t *aj;
            if (a) aj = a + ((size_t)j * LL + g) * N;
            else { or_expand_a(seed, j, g, mt, P->logN, rounds, ak); aj = ak; }
            for (uint32_t n = 0; n < N; n++) {
                ob[n] = addm(ob[n], mulm(e[n], bj[n], mt), mt);
                oa[n] = addm(oa[n], mulm(e[n], aj[n], mt), mt);
            }
        }
    }
    free(ak);
    return 0;
}

/* ------------------------------------------------------------------ */
/* ModDown                                                             */
/* ------------------------------------------------------------------ */
/* For each half h: the alpha P-limbs to coefficient form,
 *   y_p = x_p * [Phat_p^-1]_p mod p,
 *   z_i = (sum_p y_p * [Phat_p]_{q_i}) mod q_i,  Z_i = NTT_{q_i}(z_i),
 *   out_h[i] = (acc_h[i] - Z_i) * [P^-1]_{q_i} mod q_i.
 * acc: [2][l+alpha][N]; out: [2][l][N]. No rounding term (spec v1). */
int or_moddown(const or_params *P, const uint32_t *acc, uint32_t l, uint32_t *out) {
    if (check_params(P, l)) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, ll = l + al;
    uint32_t *y = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)al * N);
    uint32_t *z = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (uint32_t h = 0; h < 2; h++) {
        const uint32_t *A = acc + (size_t)h * ll * N;
        for (uint32_t k = 0; k < al; k++) {
            uint32_t pk = P->p[k], ph = 1;
            for (uint32_t m = 0; m < al; m++)
                if (m != k) ph = mulm(ph, P->p[m] % pk, pk);
            uint32_t phinv = invm(ph, pk);
            uint32_t *yk = y + (size_t)k * N;
            memcpy(yk, A + (size_t)(l + k) * N, sizeof(uint32_t) * N);
            or_ntt_inv(yk, P->logN, pk, or_min_psi(pk, P->logN));
            for (uint32_t n = 0; n < N; n++) yk[n] = mulm(yk[n], phinv, pk);
        }
        for (uint32_t i = 0; i < l; i++) {
            uint32_t qi = P->q[i];
            for (uint32_t n = 0; n < N; n++) z[n] = 0;
            for (uint32_t k = 0; k < al; k++) {
                uint32_t ph = 1; /* Phat_k mod q_i */
                for (uint32_t m = 0; m < al; m++)
                    if (m != k) ph = mulm(ph, P->p[m] % qi, qi);
                for (uint32_t n = 0; n < N; n++)
                    z[n] = addm(z[n], mulm(y[(size_t)k * N + n] % qi, ph, qi), qi);
            }
            or_ntt_fwd(z, P->logN, qi, or_min_psi(qi, P->logN));
            uint32_t pmod = 1;
            for (uint32_t k = 0; k < al; k++) pmod = mulm(pmod, P->p[k] % qi, qi);
            uint32_t pinv = invm(pmod, qi);
            uint32_t *o = out + ((size_t)h * l + i) * N;
            const uint32_t *Ai = A + (size_t)i * N;
            for (uint32_t n = 0; n < N; n++) o[n] = mulm(subm(Ai[n], z[n], qi), pinv, qi);
        }
    }
    free(z);
    free(y);
    return 0;
}

/* ------------------------------------------------------------------ */
/* full key switch                                                     */
/* ------------------------------------------------------------------ */
/* (c0, c1) decrypting under s' at level l  ->  (c0', c1') under s:
 *   ext = ModUp(c1); acc = inner(ext, ksk); (ob, oa) = ModDown(acc);
 *   c0' = c0 + ob, c1' = oa   (all mod q_i, NTT domain, canonical). */
int or_keyswitch(const or_params *P, const uint32_t *c0, const uint32_t *c1, uint32_t l,
                 const uint8_t seed[32], const uint32_t *b, const uint32_t *a, int rounds,
                 uint32_t *c0o, uint32_t *c1o) {
    if (check_params(P, l)) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, beta = (l + al - 1) / al, ll = l + al;
    uint32_t *ext = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)beta * ll * N);
    uint32_t *acc = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)2 * ll * N);
    uint32_t *out = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)2 * l * N);
    int rc = or_modup(P, c1, l, ext);
    if (!rc) rc = or_inner(P, ext, l, seed, b, a, rounds, acc);
    if (!rc) rc = or_moddown(P, acc, l, out);
    if (!rc) {
        for (uint32_t i = 0; i < l; i++) {
            uint32_t qi = P->q[i];
            for (uint32_t n = 0; n < N; n++) {
                size_t o = (size_t)i * N + n;
                c0o[o] = addm(c0[o], out[o], qi);
                c1o[o] = out[(size_t)l * N + o];
            }
        }
    }
    free(out);
    free(acc);
    free(ext);
    return rc;
}

/* ------------------------------------------------------------------ */
/* rotations (automorphism X -> X^g followed by a key switch)          */
/* ------------------------------------------------------------------ */
/* NTT-domain automorphism: slot k of the forward transform holds
 * a(psi^(2 brv(k) + 1)), so slot k of NTT(a(X^g)) is a(psi^(g (2 brv(k) + 1))),
 * the slot k' of NTT(a) with 2 brv(k') + 1 = g (2 brv(k) + 1) mod 2N.
 * g odd; one limb of N words. */
void or_automorph_ntt(const uint32_t *in, uint32_t logN, uint32_t g, uint32_t *out) {
    uint32_t N = 1u << logN;
    uint64_t twoN = 2ull * N;
    for (uint32_t k = 0; k < N; k++) {
        uint64_t e = ((2ull * bitrev(k, logN) + 1) * g) % twoN;
        uint32_t kp = bitrev((uint32_t)((e - 1) / 2), logN);
        out[k] = in[kp];
    }
}

/* Rotation of (c0, c1) (decrypting under s) by the Galois element g:
 * (c0(X^g), c1(X^g)) decrypts under s(X^g); key switch it with a key for
 * s(X^g) -> s.  The automorphism is applied to the input limbs first. */
int or_rotate(const or_params *P, const uint32_t *c0, const uint32_t *c1, uint32_t l, uint32_t g,
              const uint8_t seed[32], const uint32_t *b, const uint32_t *a, int rounds,
              uint32_t *c0o, uint32_t *c1o) {
    if (check_params(P, l) || (g & 1u) == 0 || g >= (2u << P->logN)) return -1;
    uint32_t N = 1u << P->logN;
    uint32_t *r0 = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)l * N);
    uint32_t *r1 = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)l * N);
    for (uint32_t i = 0; i < l; i++) {
        or_automorph_ntt(c0 + (size_t)i * N, P->logN, g, r0 + (size_t)i * N);
        or_automorph_ntt(c1 + (size_t)i * N, P->logN, g, r1 + (size_t)i * N);
    }
    int rc = or_keyswitch(P, r0, r1, l, seed, b, a, rounds, c0o, c1o);
    free(r1);
    free(r0);
    return rc;
}

/* One rotation of a hoisted batch: ext = ModUp(c1) is computed once for all
 * rotations of the same ciphertext; this rotation applies the automorphism to
 * every limb of ext (it commutes with the inner product and ModDown, and a
 * permuted lift is still a lift of c1(X^g)), then finishes like a key switch
 * with c0(X^g). */
int or_rotate_hoisted_one(const or_params *P, const uint32_t *c0, const uint32_t *ext, uint32_t l,
                          uint32_t g, const uint8_t seed[32], const uint32_t *b, const uint32_t *a,
                          int rounds, uint32_t *c0o, uint32_t *c1o) {
    if (check_params(P, l) || (g & 1u) == 0 || g >= (2u << P->logN)) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, beta = (l + al - 1) / al, ll = l + al;
    uint32_t *er = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)beta * ll * N);
    uint32_t *acc = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)2 * ll * N);
    uint32_t *out = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)2 * l * N);
    uint32_t *r0 = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (size_t m = 0; m < (size_t)beta * ll; m++) or_automorph_ntt(ext + m * N, P->logN, g, er + m * N);
    int rc = or_inner(P, er, l, seed, b, a, rounds, acc);
    if (!rc) rc = or_moddown(P, acc, l, out);
    if (!rc) {
        for (uint32_t i = 0; i < l; i++) {
            uint32_t qi = P->q[i];
            or_automorph_ntt(c0 + (size_t)i * N, P->logN, g, r0);
            for (uint32_t n = 0; n < N; n++) {
                size_t o = (size_t)i * N + n;
                c0o[o] = addm(r0[n], out[o], qi);
                c1o[o] = out[(size_t)l * N + o];
            }
        }
    }
    free(r0);
    free(out);
    free(acc);
    free(er);
    return rc;
}

/* ------------------------------------------------------------------ */
/* relinearisation (ciphertext product)                                */
/* ------------------------------------------------------------------ */
/* Tensor of two ciphertexts (x0, x1), (y0, y1) at level l, NTT domain, where
 * the ring product is the slot-wise product:
 *   d0 = x0 y0,  d1 = x0 y1 + x1 y0,  d2 = x1 y1      (d0 + d1 s + d2 s^2)
 * then d2 is key-switched with a key for s^2 -> s:
 *   c0' = d0 + ModDown_b,  c1' = d1 + ModDown_a. */
int or_tensor(const or_params *P, const uint32_t *x0, const uint32_t *x1, const uint32_t *y0,
              const uint32_t *y1, uint32_t l, uint32_t *d0, uint32_t *d1, uint32_t *d2) {
    if (check_params(P, l)) return -1;
    uint32_t N = 1u << P->logN;
    for (uint32_t i = 0; i < l; i++) {
        uint32_t q = P->q[i];
        for (uint32_t n = 0; n < N; n++) {
            size_t o = (size_t)i * N + n;
            d0[o] = mulm(x0[o], y0[o], q);
            d1[o] = addm(mulm(x0[o], y1[o], q), mulm(x1[o], y0[o], q), q);
            d2[o] = mulm(x1[o], y1[o], q);
        }
    }
    return 0;
}

int or_relinearize(const or_params *P, const uint32_t *x0, const uint32_t *x1, const uint32_t *y0,
                   const uint32_t *y1, uint32_t l, const uint8_t seed[32], const uint32_t *b,
                   const uint32_t *a, int rounds, uint32_t *c0o, uint32_t *c1o) {
    if (check_params(P, l)) return -1;
    uint32_t N = 1u << P->logN;
    size_t lN = (size_t)l * N;
    uint32_t *d = (uint32_t *)malloc(sizeof(uint32_t) * 3 * lN);
    uint32_t *k0 = (uint32_t *)malloc(sizeof(uint32_t) * lN);
    int rc = or_tensor(P, x0, x1, y0, y1, l, d, d + lN, d + 2 * lN);
    /* key switch of (0, d2): c0' = d0 + ob, c1' = d1 + oa */
    if (!rc) {
        memset(k0, 0, sizeof(uint32_t) * lN);
        rc = or_keyswitch(P, k0, d + 2 * lN, l, seed, b, a, rounds, c0o, c1o);
    }
    if (!rc) {
        for (uint32_t i = 0; i < l; i++) {
            uint32_t q = P->q[i];
            for (uint32_t n = 0; n < N; n++) {
                size_t o = (size_t)i * N + n;
                c0o[o] = addm(c0o[o], d[o], q);
                c1o[o] = addm(c1o[o], d[lN + o], q);
            }
        }
    }
    free(k0);
    free(d);
    return rc;
}

/* ------------------------------------------------------------------ */
/* baby-step giant-step linear transform                               */
/* ------------------------------------------------------------------ */
/* The homomorphic linear transform of CKKS bootstrapping's
 * CoeffsToSlots / SlotsToCoeffs steps by the diagonal method with baby steps
 * and giant steps (Halevi-Shoup diagonals; baby-step giant-step split as in
 * Han-Ki 2020 and Chen-Chillotti-Song 2019), with hoisted baby steps:
 *   bs_0 = (c0, c1);  bs_j = hoisted rotation of (c0, c1) by gb[j-1], j < n1
 *                           (one ModUp of c1 shared by every baby step)
 *   W_i  = sum_{j<n1} diag[i][j] (.) bs_j      (slot-wise, both halves)
 *   out  = W_0 + sum_{1<=i<n2} rotation of W_i by gg[i-1]
 * diag: [n2][n1][l][N] NTT-domain plaintexts (the caller's pre-rotated
 * diagonals); baby key j-1 (seed_b + 32 (j-1), b_b[j-1]) switches
 * s(X^gb[j-1]) -> s, giant key i-1 switches s(X^gg[i-1]) -> s.  The 'a'
 * halves are regenerated (rounds).  out0, out1: [l][N]. */
int or_linear_transform(const or_params *P, const uint32_t *c0, const uint32_t *c1, uint32_t l,
                        uint32_t n1, const uint32_t *gb, const uint8_t *seed_b, const uint32_t *const *b_b,
                        uint32_t n2, const uint32_t *gg, const uint8_t *seed_g, const uint32_t *const *b_g,
                        const uint32_t *diag, int rounds, uint32_t *out0, uint32_t *out1) {
    if (check_params(P, l) || n1 < 1 || n2 < 1) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, beta = (l + al - 1) / al, ll = l + al;
    size_t lN = (size_t)l * N;
    uint32_t *ext = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)beta * ll * N);
    uint32_t *bs = (uint32_t *)malloc(sizeof(uint32_t) * 2 * lN * n1);
    uint32_t *w = (uint32_t *)malloc(sizeof(uint32_t) * 2 * lN);
    uint32_t *r = (uint32_t *)malloc(sizeof(uint32_t) * 2 * lN);
    int rc = or_modup(P, c1, l, ext);
    /* baby steps */
    memcpy(bs, c0, sizeof(uint32_t) * lN);
    memcpy(bs + lN, c1, sizeof(uint32_t) * lN);
    for (uint32_t j = 1; j < n1 && !rc; j++)
        rc = or_rotate_hoisted_one(P, c0, ext, l, gb[j - 1], seed_b + 32 * (size_t)(j - 1), b_b[j - 1], NULL,
                                   rounds, bs + 2 * lN * j, bs + 2 * lN * j + lN);
    /* giant steps */
    for (uint32_t i = 0; i < n2 && !rc; i++) {
        for (uint32_t t = 0; t < l; t++) {
            uint32_t q = P->q[t];
            for (uint32_t n = 0; n < N; n++) {
                size_t o = (size_t)t * N + n;
                uint32_t v0 = 0, v1 = 0;
                for (uint32_t j = 0; j < n1; j++) {
                    uint32_t d = diag[((size_t)i * n1 + j) * lN + o];
                    v0 = addm(v0, mulm(d, bs[2 * lN * j + o], q), q);
                    v1 = addm(v1, mulm(d, bs[2 * lN * j + lN + o], q), q);
                }
                w[o] = v0;
                w[lN + o] = v1;
            }
        }
        if (i == 0) {
            memcpy(out0, w, sizeof(uint32_t) * lN);
            memcpy(out1, w + lN, sizeof(uint32_t) * lN);
            continue;
        }
        rc = or_rotate(P, w, w + lN, l, gg[i - 1], seed_g + 32 * (size_t)(i - 1), b_g[i - 1], NULL, rounds, r,
                       r + lN);
        for (uint32_t t = 0; t < l && !rc; t++) {
            uint32_t q = P->q[t];
            for (uint32_t n = 0; n < N; n++) {
                size_t o = (size_t)t * N + n;
                out0[o] = addm(out0[o], r[o], q);
                out1[o] = addm(out1[o], r[lN + o], q);
            }
        }
    }
    free(r);
    free(w);
    free(bs);
    free(ext);
    return rc;
}

/* ------------------------------------------------------------------ */
/* key generation (the oracle side only; the library never generates)  */
/* ------------------------------------------------------------------ */

/* integer polynomial -> residues mod q */
static void reduce_poly(const int64_t *s, uint32_t N, uint32_t q, uint32_t *out) {
    for (uint32_t n = 0; n < N; n++) {
        int64_t v = s[n] % (int64_t)q;
        if (v < 0) v += q;
        out[n] = (uint32_t)v;
    }
}

/* Negacyclic schoolbook product of integer polynomials (mod X^N + 1),
 * exact in int64 for the small-coefficient inputs it is used on. */
void or_negacyclic_mul(const int64_t *a, const int64_t *b, uint32_t logN, int64_t *out) {
    uint32_t N = 1u << logN;
    for (uint32_t k = 0; k < N; k++) out[k] = 0;
    for (uint32_t i = 0; i < N; i++) {
        if (a[i] == 0) continue;
        for (uint32_t j = 0; j < N; j++) {
            uint32_t k = i + j;
            if (k < N) out[k] += a[i] * b[j];
            else out[k - N] -= a[i] * b[j];
        }
    }
}

/* s(X) -> s(X^g) mod X^N + 1 for odd g: coefficient n moves to n*g mod 2N,
 * negated when that lands at or above N (X^N = -1). */
void or_automorph(const int64_t *s, uint32_t logN, uint32_t g, int64_t *out) {
    uint32_t N = 1u << logN;
    uint64_t twoN = 2ull * N;
    for (uint32_t n = 0; n < N; n++) out[n] = 0;
    for (uint32_t n = 0; n < N; n++) {
        uint64_t m = ((uint64_t)n * g) % twoN;
        if (m < N) out[m] += s[n];
        else out[m - N] -= s[n];
    }
}

/* Key-switching key for s' -> s, 'b' half, NTT domain, [dnum][L+alpha][N]:
 *   b_{j,g} = -a_{j,g} * s_hat + e_j_hat + [P]_{q_g} * s'_hat * [q_g in D_j]
 * with D_j the top-level digit {q_{j*alpha}..q_{min(j*alpha+alpha,L)-1}}
 * (gadget 1 on the digit, 0 on the other q's; the P-limbs carry no s' term),
 * a_{j,g} from or_expand_a.  s, s': integer coefficient vectors; e: [dnum][N]. */
int or_ksk_gen(const or_params *P, const int64_t *s, const int64_t *sp, const int64_t *e,
               const uint8_t seed[32], int rounds, uint32_t *b) {
    if (check_params(P, P->L)) return -1;
    uint32_t N = 1u << P->logN, al = P->alpha, LL = P->L + al;
    uint32_t *sh = (uint32_t *)malloc(sizeof(uint32_t) * N);
    uint32_t *sph = (uint32_t *)malloc(sizeof(uint32_t) * N);
    uint32_t *eh = (uint32_t *)malloc(sizeof(uint32_t) * N);
    uint32_t *ak = (uint32_t *)malloc(sizeof(uint32_t) * N);
    for (uint32_t g = 0; g < LL; g++) {
        uint32_t q = prime_of(P, g), psi = or_min_psi(q, P->logN);
        reduce_poly(s, N, q, sh);
        or_ntt_fwd(sh, P->logN, q, psi);
        reduce_poly(sp, N, q, sph);
        or_ntt_fwd(sph, P->logN, q, psi);
        uint32_t pm = 1;
        for (uint32_t k = 0; k < al; k++) pm = mulm(pm, P->p[k] % q, q);
        for (uint32_t j = 0; j < P->dnum; j++) {
            reduce_poly(e + (size_t)j * N, N, q, eh);
            or_ntt_fwd(eh, P->logN, q, psi);
            or_expand_a(seed, j, g, q, P->logN, rounds, ak);
            int in_digit = (g < P->L) && (g >= j * al) && (g < j * al + al);
            uint32_t *bj = b + ((size_t)j * LL + g) * N;
            for (uint32_t n = 0; n < N; n++) {
                uint32_t v = subm(eh[n], mulm(ak[n], sh[n], q), q);
                if (in_digit) v = addm(v, mulm(pm, sph[n], q), q);
                bj[n] = v;
            }
        }
    }
    free(ak);
    free(eh);
    free(sph);
    free(sh);
    return 0;
}
