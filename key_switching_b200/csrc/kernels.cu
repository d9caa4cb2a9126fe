// kernels.cu -- the key-switching kernels for sm_100a and their launchers.
//
// Dataflow of one key switch at level l (hybrid key switching, Han-Ki 2020;
// full-RNS CKKS, Cheon et al. 2018), with N = R x C (rows of C words):
//   k_row(inv)         c1 rows: inverse row pass                 -> W1
//   k_col(inv,scale)   W1 columns: inverse column pass, times
//                      N^-1 [Dhat_i^-1]_{q_i}                     -> y (in W1)
//   k_bconv_col(ModUp) per digit j and target t outside D_j:
//                      z_t = sum_i y_i [Dhat_i]_t, forward column pass -> T[j][t]
//   k_inner            per target limb t: forward row pass of T[j][t] (or the
//                      input limb when t is in D_j), times b_{j,t} and the
//                      ChaCha12-regenerated a_{j,t}, summed over j; the
//                      special-prime limbs then get the inverse row pass -> ACC
//   k_col(inv,scale)   ACC special limbs: inverse column pass, times
//                      N^-1 [Phat_p^-1]_p                         -> y_P (in ACC)
//   k_bconv_col(ModDown) z_i = sum_p y_p [Phat_p]_{q_i}, forward column pass -> U
//   k_moddown_row      forward row pass of U, (acc - z) [P^-1]_{q_i} (+ c0) -> out
// Values between passes are lazy ([0, 2q)); every stored result of an ABI call
// is canonical.
#include <cuda_runtime.h>

#include <type_traits>

#include "chacha.cuh"
#include "ntt.cuh"
#include "pc_internal.h"

namespace pc {

// ------------------------------------------------------------------ helpers

// global prime index of local limb t at level l
__device__ __forceinline__ u32 glob_of(const Tables &T, u32 l, u32 t) {
    return t < l ? t : T.L + (t - l);
}

// Load / store the 16 registers of a phase layout from / to a line in global
// memory.  Runs of >= 4 consecutive elements (distance-1 phases) use 16-byte
// accesses; the others are scalar and coalesced across the line's threads.
template <class PH>
__device__ __forceinline__ void gload(u32 v[16], const u32 *line, int lt) {
    if constexpr (PH::D == 1 && PH::KK >= 4) {
#pragma unroll
        for (int r = 0; r < 16; r += 4) {
            uint4 t = *reinterpret_cast<const uint4 *>(line + PH::x_of(lt, r));
            v[r] = t.x; v[r + 1] = t.y; v[r + 2] = t.z; v[r + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = line[PH::x_of(lt, r)];
    }
}
template <class PH>
__device__ __forceinline__ void gstore(const u32 v[16], u32 *line, int lt) {
    if constexpr (PH::D == 1 && PH::KK >= 4) {
#pragma unroll
        for (int r = 0; r < 16; r += 4)
            *reinterpret_cast<uint4 *>(line + PH::x_of(lt, r)) = make_uint4(v[r], v[r + 1], v[r + 2], v[r + 3]);
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) line[PH::x_of(lt, r)] = v[r];
    }
}

// phase that holds the registers at the end of a forward line transform
template <int LOGM>
struct LastPhase {
    using PL = Plan<LOGM>;
    using type = typename std::conditional<
        PL::NPH == 1, typename PL::P0,
        typename std::conditional<PL::NPH == 2, typename PL::P1, typename PL::P2>::type>::type;
};

struct RowAddr {
    __device__ __forceinline__ int operator()(int x) const { return x + (x >> 4); }
};
template <int LS>
struct ColAddr {
    int c;
    __device__ __forceinline__ int operator()(int x) const { return x * LS + c; }
};
struct TwGlobal {
    const uint2 *t;
    __device__ __forceinline__ uint2 operator()(int i) const { return __ldg(t + i); }
};
struct TwShared {
    const uint2 *t;
    __device__ __forceinline__ uint2 operator()(int i) const { return t[i]; }
};

// ------------------------------------------------------------------ row pass
// grid (ROW_BLOCKS, nlimbs, Z).  In place allowed (in == out).
template <int LOGN, bool FWD>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS)
k_row(Tables T, const u32 *in, u32 *out, u32 first_prime, size_t zin, size_t zout, int canonical) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    __shared__ u32 sm[GE::NL * GE::ROW_LS];
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row = blockIdx.x * GE::NL + rho;
    const u32 g = first_prime + blockIdx.y;
    const u32 q = T.pk[g].q;
    const size_t off = (size_t)blockIdx.y * GE::N + (size_t)row * GE::C;
    const u32 *src = in + blockIdx.z * zin + off;
    u32 *dst = out + blockIdx.z * zout + off;
    u32 v[16];
    u32 *line = sm + rho * GE::ROW_LS;
    if constexpr (FWD) {
        gload<PF>(v, src, lt);
        line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, TwGlobal{T.rowF + (size_t)g * GE::N + (size_t)row * GE::C}, q);
        if (canonical) {
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = red1(v[r], q);
        }
        gstore<PLAST>(v, dst, lt);
    } else {
        gload<PLAST>(v, src, lt);
        line_inv<GE::LOGC>(v, line, lt, RowAddr{}, TwGlobal{T.rowI + (size_t)g * GE::N + (size_t)row * GE::C}, q);
        if (canonical) {
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = red1(v[r], q);
        }
        gstore<PF>(v, dst, lt);
    }
}

// --------------------------------------------------------------- column pass
// grid (COL_BLOCKS, nlimbs, Z).  In place allowed.  scale_mode: 0 none (lazy
// out), 1 N^-1, 2 ModUp digit scale at level l, 3 ModDown P-hat scale.
template <int LOGN, bool FWD>
__global__ void __launch_bounds__(Geo<LOGN>::COL_THREADS)
k_col(Tables T, const u32 *in, u32 *out, u32 first_prime, size_t zin, size_t zout, int scale_mode,
      u32 l) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    __shared__ u32 sm[GE::R * GE::COL_LS];
    __shared__ uint2 tw[GE::R];
    const int c = threadIdx.x % GE::W, lt = threadIdx.x / GE::W;
    const int col = blockIdx.x * GE::W + c;
    const u32 k = blockIdx.y, g = first_prime + k;
    const u32 q = T.pk[g].q;
    const uint2 *tab = (FWD ? T.colF : T.colI) + (size_t)g * GE::R;
    for (int i = threadIdx.x; i < GE::R; i += GE::COL_THREADS) tw[i] = tab[i];
    const size_t off = (size_t)k * GE::N + col;
    const u32 *src = in + blockIdx.z * zin + off;
    u32 *dst = out + blockIdx.z * zout + off;
    u32 v[16];
    __syncthreads();
    if constexpr (FWD) {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = src[(size_t)PF::x_of(lt, r) * GE::C];
        line_fwd<GE::LOGR>(v, sm, lt, ColAddr<GE::COL_LS>{c}, TwShared{tw}, q);
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PLAST::x_of(lt, r) * GE::C] = v[r];
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = src[(size_t)PLAST::x_of(lt, r) * GE::C];
        line_inv<GE::LOGR>(v, sm, lt, ColAddr<GE::COL_LS>{c}, TwShared{tw}, q);
        uint2 s = make_uint2(0, 0);
        if (scale_mode == 1) s = make_uint2(T.pk[g].ninv, T.pk[g].ninvs);
        else if (scale_mode == 2) {
            const u32 j = k / T.alpha, d = min(T.alpha, l - j * T.alpha);
            s = T.upScale[(size_t)(d - 1) * T.L + k];
        } else if (scale_mode == 3) s = T.downScale[g - T.L];
        if (scale_mode) {
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = shoup(v[r], s.x, s.y, q);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PF::x_of(lt, r) * GE::C] = v[r];
    }
}

// ------------------------------------------- basis conversion + column pass
// grid (COL_BLOCKS, target groups, units * Z); blockIdx.z = z * units + unit.
// ModUp (mode 0): unit = digit j; sources y_i, i in D_j (limbs of y);
//   targets: local t in [0, l+alpha) \ D_j -> out[j][t] ([beta][l+alpha][N]).
// ModDown (mode 1): unit = half h; sources = the alpha special limbs of ACC
//   half h (already y_p); targets i < l -> out[h][i] ([2][l][N]).
// out[t] = forward column pass of z_t = sum_k y_k c_{k,t} mod t (lazy).
template <int LOGN>
__global__ void __launch_bounds__(Geo<LOGN>::COL_THREADS)
k_bconv_col(Tables T, int mode, const u32 *y, size_t yz, u32 *out, size_t outz, u32 l, u32 tg_size) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    extern __shared__ __align__(16) u32 dyn[];
    u32 *sy = dyn;                                   // [d][R][W]
    u32 *sx = dyn + T.alpha * GE::R * GE::W;         // [R][W+1]
    uint2 *tw = reinterpret_cast<uint2 *>(sx + GE::R * GE::COL_LS);  // [R]
    const int c = threadIdx.x % GE::W, lt = threadIdx.x / GE::W;
    const int col0 = blockIdx.x * GE::W;
    const u32 units = mode == 0 ? (l + T.alpha - 1) / T.alpha : 2;
    const u32 z = blockIdx.z / units, unit = blockIdx.z % units;
    const u32 ll = l + T.alpha;
    u32 d, ntarg;
    const u32 *ysrc;
    if (mode == 0) {
        d = min(T.alpha, l - unit * T.alpha);
        ntarg = ll - d;
        ysrc = y + z * yz + (size_t)unit * T.alpha * GE::N;
    } else {
        d = T.alpha;
        ntarg = l;
        ysrc = y + z * yz + ((size_t)unit * ll + l) * GE::N;
    }
    const u32 t0 = blockIdx.y * tg_size;
    if (t0 >= ntarg) return;
    const u32 t1 = min(t0 + tg_size, ntarg);
    // stage the source tile [d][R][W]
    for (u32 e = threadIdx.x; e < d * GE::R * GE::W; e += GE::COL_THREADS) {
        const u32 k = e / (GE::R * GE::W), rem = e % (GE::R * GE::W);
        const u32 x = rem / GE::W, cc = rem % GE::W;
        sy[e] = ysrc[(size_t)k * GE::N + (size_t)x * GE::C + col0 + cc];
    }
    for (u32 ti = t0; ti < t1; ++ti) {
        u32 g;
        const u32 *conv;
        u32 *dst;
        if (mode == 0) {
            const u32 lo = unit * T.alpha;
            const u32 t = ti < lo ? ti : ti + d;
            g = glob_of(T, l, t);
            conv = T.upConv + (((size_t)unit * T.alpha + (d - 1)) * T.NP + g) * T.alpha;
            dst = out + z * outz + ((size_t)unit * ll + t) * GE::N;
        } else {
            g = ti;
            conv = T.downConv + (size_t)ti * T.alpha;
            dst = out + z * outz + ((size_t)unit * l + ti) * GE::N;
        }
        const PrimeK pk = T.pk[g];
        __syncthreads();  // previous target's readers of tw / sx are done
        for (int i = threadIdx.x; i < GE::R; i += GE::COL_THREADS) tw[i] = T.colF[(size_t)g * GE::R + i];
        u32 cv[MAX_ALPHA];
#pragma unroll
        for (int k = 0; k < MAX_ALPHA; ++k) cv[k] = (k < (int)d) ? __ldg(conv + k) : 0u;
        __syncthreads();
        u32 v[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int x = PF::x_of(lt, r);
            u64 s = 0;
#pragma unroll
            for (int k = 0; k < MAX_ALPHA; ++k) {
                if (k < (int)d) {
                    if (k == 4 || k == 6) s = fold64(s, pk.q, pk.q1s);
                    s += (u64)sy[(k * GE::R + x) * GE::W + c] * cv[k];
                }
            }
            v[r] = redc64(s, pk.q, pk.qn, pk.q1s);
        }
        line_fwd<GE::LOGR>(v, sx, lt, ColAddr<GE::COL_LS>{c}, TwShared{tw}, pk.q);
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PLAST::x_of(lt, r) * GE::C + col0 + c] = v[r];
    }
}

// ------------------------------------------------------------- inner product
// grid (ROW_BLOCKS, l+alpha, Z).  For target limb t, sum over digits j of
// ext_j[t] * (b, a)_{j,g(t)}.  FUSED: ext_j[t] = forward row pass of the
// column-pass output src[j][t] (or c1[t] for t in D_j); else ext = src.
// REGEN: a from ChaCha12 (spec v1), else from the stored key.
// PINTT: special-prime limbs get the inverse row pass before the store.
template <int LOGN, bool FUSED, bool REGEN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS)
k_inner(Tables T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z, u32 *acc, size_t accz,
        u32 l, KeyPack kp, int pintt) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    __shared__ u32 sm[GE::NL * GE::ROW_LS];
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row = blockIdx.x * GE::NL + rho;
    const u32 t = blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    const size_t rowoff = (size_t)row * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    u32 seed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) seed[i] = kp.seed[z][i];
    const u32 *kb = kp.b[z];
    const u32 *ka = kp.a[z];
    const size_t LLN = (size_t)(T.L + T.alpha) * GE::N;

    u64 sb[16], sa[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) { sb[r] = 0; sa[r] = 0; }

    for (u32 j = 0; j < beta; ++j) {
        u32 v[16];
        const bool own = (t < l) && (t / T.alpha == j);
        if (FUSED && !own) {
            gload<PF>(v, src + z * srcz + ((size_t)j * ll + t) * GE::N + rowoff, lt);
            line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, TwGlobal{T.rowF + (size_t)g * GE::N + rowoff}, q);
        } else if (FUSED) {
            gload<PLAST>(v, c1 + z * c1z + (size_t)t * GE::N + rowoff, lt);
        } else {
            gload<PLAST>(v, src + z * srcz + ((size_t)j * ll + t) * GE::N + rowoff, lt);
        }
        u32 bv[16];
        gload<PLAST>(bv, kb + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        u32 av[16];
        if constexpr (REGEN) {
            // the thread's elements form groups of KK consecutive coefficients
#pragma unroll
            for (int gi = 0; gi < PLAST::G; ++gi) {
                const u32 base = (u32)(rowoff + PLAST::x_of(lt, gi * PLAST::KK));
#pragma unroll
                for (int bb = 0; bb < (PLAST::KK + 7) / 8; ++bb) {
                    u32 ks[16];
                    const u32 k0 = base + bb * 8;
                    chacha12_block(seed, k0 >> 3, g, j, ks);
#pragma unroll
                    for (int w = 0; w < 8 && bb * 8 + w < PLAST::KK; ++w) {
                        const u32 wi = (k0 + w) & 7;
                        const u32 lo = ks[2 * wi], hi = ks[2 * wi + 1];
                        // a * 2^-32 mod q
                        av[gi * PLAST::KK + bb * 8 + w] = redc(lo, mod32(hi, q, pk.q1s), q, pk.qn);
                    }
                }
            }
        } else {
            gload<PLAST>(av, ka + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        }
        const bool fold = (j & 1) && (j + 1 < beta);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const u32 e = red1(v[r], q);
            sb[r] += (u64)e * bv[r];
            sa[r] += (u64)e * av[r];
            if (fold) {
                sb[r] = fold64(sb[r], q, pk.q1s);
                sa[r] = fold64(sa[r], q, pk.q1s);
            }
        }
    }
    // canonical sums: REDC divides by 2^32; regenerated a carries another 2^-32
    u32 ob[16], oa[16];
    const u32 ca = REGEN ? pk.r64 : pk.r32, cas = REGEN ? pk.r64s : pk.r32s;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        ob[r] = shoup(redc64(sb[r], q, pk.qn, pk.q1s), pk.r32, pk.r32s, q);
        oa[r] = shoup(redc64(sa[r], q, pk.qn, pk.q1s), ca, cas, q);
    }
    u32 *d0 = acc + z * accz + (size_t)t * GE::N + rowoff;
    u32 *d1 = acc + z * accz + (size_t)(ll + t) * GE::N + rowoff;
    if (pintt && t >= l) {
        const TwGlobal twi{T.rowI + (size_t)g * GE::N + rowoff};
        line_inv<GE::LOGC>(ob, line, lt, RowAddr{}, twi, q);
        gstore<PF>(ob, d0, lt);
        line_inv<GE::LOGC>(oa, line, lt, RowAddr{}, twi, q);
        gstore<PF>(oa, d1, lt);
    } else {
        gstore<PLAST>(ob, d0, lt);
        gstore<PLAST>(oa, d1, lt);
    }
}

// ----------------------------------------------------------- ModDown finish
// grid (ROW_BLOCKS, l, Z).  out_h[i] = (acc_h[i] - rowfwd(U_h[i])) [P^-1]_{q_i},
// plus c0 for h = 0 when c0 is given.  out0/out1 may alias c0 / the input.
template <int LOGN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS)
k_moddown_row(Tables T, const u32 *U, size_t Uz, const u32 *acc, size_t accz, const u32 *c0,
              size_t c0z, u32 *out0, u32 *out1, size_t outz, u32 l) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    __shared__ u32 sm[GE::NL * GE::ROW_LS];
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row = blockIdx.x * GE::NL + rho;
    const u32 i = blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha;
    const PrimeK pk = T.pk[i];
    const u32 q = pk.q;
    const uint2 pinv = T.pInv[i];
    const size_t rowoff = (size_t)row * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwGlobal tw{T.rowF + (size_t)i * GE::N + rowoff};
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        u32 v[16], a[16];
        gload<PF>(v, U + z * Uz + ((size_t)h * l + i) * GE::N + rowoff, lt);
        line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q);
        gload<PLAST>(a, acc + z * accz + ((size_t)h * ll + i) * GE::N + rowoff, lt);
        u32 o[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) o[r] = shoup(a[r] - red1(v[r], q) + q, pinv.x, pinv.y, q);
        if (h == 0 && c0) {
            u32 cc[16];
            gload<PLAST>(cc, c0 + z * c0z + (size_t)i * GE::N + rowoff, lt);
#pragma unroll
            for (int r = 0; r < 16; ++r) o[r] = red1(o[r] + cc[r], q);
        }
        gstore<PLAST>(o, (h == 0 ? out0 : out1) + z * outz + (size_t)i * GE::N + rowoff, lt);
    }
}

// ------------------------------------------------------------ ModUp finish
// grid (ROW_BLOCKS, l+alpha, beta).  ext[j][t] = c1[t] for t in D_j, else the
// forward row pass (in place) of the column-pass output already in ext[j][t].
template <int LOGN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS)
k_modup_finish(Tables T, const u32 *c1, u32 *ext, u32 l) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    __shared__ u32 sm[GE::NL * GE::ROW_LS];
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row = blockIdx.x * GE::NL + rho;
    const u32 t = blockIdx.y, j = blockIdx.z;
    const u32 ll = l + T.alpha;
    const u32 g = glob_of(T, l, t);
    const u32 q = T.pk[g].q;
    const size_t rowoff = (size_t)row * GE::C;
    u32 *dst = ext + ((size_t)j * ll + t) * GE::N + rowoff;
    u32 v[16];
    if (t < l && t / T.alpha == j) {
        gload<PLAST>(v, c1 + (size_t)t * GE::N + rowoff, lt);
        gstore<PLAST>(v, dst, lt);
        return;
    }
    gload<PF>(v, dst, lt);
    line_fwd<GE::LOGC>(v, sm + rho * GE::ROW_LS, lt, RowAddr{}, TwGlobal{T.rowF + (size_t)g * GE::N + rowoff}, q);
#pragma unroll
    for (int r = 0; r < 16; ++r) v[r] = red1(v[r], q);
    gstore<PLAST>(v, dst, lt);
}

// ---------------------------------------------------------- expand (test hook)
// one thread per ChaCha block: out[j][t][8b .. 8b+7]
template <int LOGN>
__global__ void k_expand(Tables T, KeyPack kp, u32 l, u32 *out) {
    constexpr int N = 1 << LOGN;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const size_t total = (size_t)beta * ll * (N / 8);
    const size_t id = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= total) return;
    const u32 blk = (u32)(id % (N / 8));
    const u32 t = (u32)((id / (N / 8)) % ll);
    const u32 j = (u32)(id / ((size_t)(N / 8) * ll));
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    u32 ks[16];
    chacha12_block(kp.seed[0], blk, g, j, ks);
    u32 *o = out + ((size_t)j * ll + t) * N + (size_t)blk * 8;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        // (hi 2^32 + lo) mod q = REDC((hi mod q) 2^32 + lo) * 2^32
        const u32 am = redc(ks[2 * w], mod32(ks[2 * w + 1], pk.q, pk.q1s), pk.q, pk.qn);
        o[w] = shoup(am, pk.r32, pk.r32s, pk.q);
    }
}

// ================================================================ launchers

#define PC_DISPATCH(LOGN_VAR, ...)                     \
    switch (LOGN_VAR) {                                \
        case 10: { constexpr int LG = 10; __VA_ARGS__; break; } \
        case 11: { constexpr int LG = 11; __VA_ARGS__; break; } \
        case 12: { constexpr int LG = 12; __VA_ARGS__; break; } \
        case 13: { constexpr int LG = 13; __VA_ARGS__; break; } \
        case 14: { constexpr int LG = 14; __VA_ARGS__; break; } \
        case 15: { constexpr int LG = 15; __VA_ARGS__; break; } \
        case 16: { constexpr int LG = 16; __VA_ARGS__; break; } \
        case 17: { constexpr int LG = 17; __VA_ARGS__; break; } \
        default: return cudaErrorInvalidValue;         \
    }

template <int LG>
static size_t bconv_smem(const pc_ctx *c) {
    using GE = Geo<LG>;
    return sizeof(u32) * ((size_t)c->alpha * GE::R * GE::W + (size_t)GE::R * GE::COL_LS + 2 * GE::R);
}

cudaError_t prepare_kernels(const pc_ctx *c) {
    PC_DISPATCH(c->logN, {
        cudaError_t e = cudaFuncSetAttribute(k_bconv_col<LG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)bconv_smem<LG>(c));
        if (e != cudaSuccess) return e;
    });
    return cudaSuccess;
}

cudaError_t launch_row(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime,
                       u32 nlimbs, u32 Z, size_t zin, size_t zout, bool canonical, cudaStream_t s) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, nlimbs, Z);
        if (fwd) k_row<LG, true><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, in, out, first_prime, zin, zout, canonical);
        else k_row<LG, false><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, in, out, first_prime, zin, zout, canonical);
    });
    return cudaGetLastError();
}

cudaError_t launch_col(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime,
                       u32 nlimbs, u32 Z, size_t zin, size_t zout, int scale_mode, u32 l,
                       cudaStream_t s) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::COL_BLOCKS, nlimbs, Z);
        if (fwd) k_col<LG, true><<<grid, GE::COL_THREADS, 0, s>>>(c->tab, in, out, first_prime, zin, zout, scale_mode, l);
        else k_col<LG, false><<<grid, GE::COL_THREADS, 0, s>>>(c->tab, in, out, first_prime, zin, zout, scale_mode, l);
    });
    return cudaGetLastError();
}

cudaError_t launch_bconv_col(const pc_ctx *c, int mode, const u32 *y, size_t yz, u32 *out,
                             size_t outz, u32 l, u32 Z, cudaStream_t s) {
    const u32 units = mode == 0 ? (l + c->alpha - 1) / c->alpha : 2;
    const u32 maxt = mode == 0 ? l + c->alpha - 1 : l;  // most targets of any unit
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        // aim for about four CTAs per SM in total
        const u64 want = 4ull * (u64)c->num_sms;
        const u64 per_tg1 = (u64)GE::COL_BLOCKS * units * Z * maxt;
        u32 tg = (u32)((per_tg1 + want - 1) / want);
        if (tg < 1) tg = 1;
        if (tg > maxt) tg = maxt;
        const u32 ntg = (maxt + tg - 1) / tg;
        dim3 grid(GE::COL_BLOCKS, ntg, units * Z);
        k_bconv_col<LG><<<grid, GE::COL_THREADS, bconv_smem<LG>(c), s>>>(c->tab, mode, y, yz, out, outz, l, tg);
    });
    return cudaGetLastError();
}

cudaError_t launch_inner(const pc_ctx *c, bool fused, const u32 *src, size_t srcz,
                         const u32 *c1, size_t c1z, u32 *acc, size_t accz, u32 l, const KeyPack &kp,
                         u32 Z, bool regen, bool pintt, cudaStream_t s) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l + c->alpha, Z);
        if (fused && regen) k_inner<LG, true, true><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else if (fused) k_inner<LG, true, false><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else if (regen) k_inner<LG, false, true><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else k_inner<LG, false, false><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
    });
    return cudaGetLastError();
}

cudaError_t launch_moddown_row(const pc_ctx *c, const u32 *U, size_t Uz, const u32 *acc,
                               size_t accz, const u32 *c0, size_t c0z, u32 *out0, u32 *out1,
                               size_t outz, u32 l, u32 Z, cudaStream_t s) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l, Z);
        k_moddown_row<LG><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, U, Uz, acc, accz, c0, c0z, out0, out1, outz, l);
    });
    return cudaGetLastError();
}

cudaError_t launch_modup_finish(const pc_ctx *c, const u32 *c1, u32 *ext, u32 l, cudaStream_t s) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l + c->alpha, (l + c->alpha - 1) / c->alpha);
        k_modup_finish<LG><<<grid, GE::ROW_THREADS, 0, s>>>(c->tab, c1, ext, l);
    });
    return cudaGetLastError();
}

cudaError_t launch_expand(const pc_ctx *c, const u32 seed[8], u32 l, u32 *out, cudaStream_t s) {
    KeyPack kp{};
    for (int i = 0; i < 8; ++i) kp.seed[0][i] = seed[i];
    const u64 total = (u64)((l + c->alpha - 1) / c->alpha) * (l + c->alpha) * (c->N / 8);
    const u32 threads = 256;
    const u32 blocks = (u32)((total + threads - 1) / threads);
    PC_DISPATCH(c->logN, { k_expand<LG><<<blocks, threads, 0, s>>>(c->tab, kp, l, out); });
    return cudaGetLastError();
}

}  // namespace pc
