// kernels.cu -- the key-switching kernels for sm_100a and their launchers.
//
// Dataflow of one key switch at level l (hybrid key switching, Han-Ki 2020;
// full-RNS CKKS, Cheon et al. 2018), with N = R x C (rows of C words):
//   k_row(inv)         c1 rows: inverse row pass                 -> W1
//   k_colconv(ModUp)   per digit j and column block, one CTA cluster:
//                      inverse column pass of the digit's limbs, times
//                      N^-1 [Dhat_i^-1]_{q_i} (y), shared over DSMEM;
//                      z_t = sum_i y_i [Dhat_i]_t for t outside D_j,
//                      forward column pass                        -> T[j][t]
//   k_inner            per target limb t: forward row pass of T[j][t] (or the
//                      input limb when t is in D_j), times b_{j,t} and the
//                      ChaCha12-regenerated a_{j,t}, summed over j; the
//                      special-prime limbs then get the inverse row pass -> ACC
//   k_colconv(ModDown) per half and column block: inverse column pass of the
//                      special limbs times N^-1 [Phat_p^-1]_p, DSMEM share,
//                      z_i = sum_p y_p [Phat_p]_{q_i}, forward column pass -> U
//   k_moddown_row      forward row pass of U, (acc - z) [P^-1]_{q_i} (+ c0) -> out
// Values between passes are lazy ([0, 2q)); every stored result of an ABI call
// is canonical.
#include <cuda_runtime.h>

#include <cooperative_groups.h>

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
template <int W>
struct ColAddr {
    int c;
    __device__ __forceinline__ int operator()(int x) const { return (x + (x >> 4)) * W + c; }
};
// Stage the re-laid row twiddle tables of this CTA's NL rows into shared
// memory with asynchronous copies (all in flight at once).  Caller waits.
template <class GE>
__device__ __forceinline__ void stage_row_tw(uint2 *stw, const uint2 *tab_rows) {
    constexpr int VEC = GE::NL * GE::C / 2;  // 16-byte chunks
#pragma unroll
    for (int i = threadIdx.x; i < VEC; i += GE::ROW_THREADS)
        cp_async16(stw + 2 * i, tab_rows + 2 * i);
}

template <class GE>
constexpr size_t row_smem_bytes() {
    return sizeof(u32) * GE::NL * GE::ROW_LS + sizeof(uint2) * GE::NL * GE::C;
}

// ------------------------------------------------------------------ row pass
// grid (ROW_BLOCKS, nlimbs, Z).  In place allowed (in == out).
template <int LOGN, bool FWD>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS)
k_row(Tables T, const u32 *in, u32 *out, u32 first_prime, size_t zin, size_t zout, int canonical) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);          // [NL][C]
    u32 *sm = dyn + 2 * GE::NL * GE::C;                      // [NL][ROW_LS]
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 g = first_prime + blockIdx.y;
    const u32 q = T.pk[g].q;
    stage_row_tw<GE>(stw, (FWD ? T.rowF : T.rowI) + (size_t)g * GE::N + (size_t)row0 * GE::C);
    pdl_wait();
    pdl_trigger();
    const size_t off = (size_t)blockIdx.y * GE::N + (size_t)row * GE::C;
    const u32 *src = in + blockIdx.z * zin + off;
    u32 *dst = out + blockIdx.z * zout + off;
    u32 v[16];
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    if constexpr (FWD) gload<PF>(v, src, lt);
    else gload<PLAST>(v, src, lt);
    cp_async_wait_all();
    __syncthreads();
    if constexpr (FWD) {
        line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
        if (canonical) {
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = red1(v[r], q);
        }
        gstore<PLAST>(v, dst, lt);
    } else {
        line_inv<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
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
    __shared__ u32 sm[GE::COL_TILE];
    __shared__ uint2 tw[GE::R];
    const int c = threadIdx.x % GE::W, lt = threadIdx.x / GE::W;
    const int col = blockIdx.x * GE::W + c;
    const u32 k = blockIdx.y, g = first_prime + k;
    const u32 q = T.pk[g].q;
    const uint2 *tab = (FWD ? T.colF : T.colI) + (size_t)g * GE::R;
    for (int i = threadIdx.x; i < GE::R; i += GE::COL_THREADS) tw[i] = tab[i];
    pdl_wait();
    pdl_trigger();
    const size_t off = (size_t)k * GE::N + col;
    const u32 *src = in + blockIdx.z * zin + off;
    u32 *dst = out + blockIdx.z * zout + off;
    u32 v[16];
    __syncthreads();
    if constexpr (FWD) {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = src[(size_t)PF::x_of(lt, r) * GE::C];
        line_fwd<GE::LOGR>(v, sm, lt, ColAddr<GE::W>{c}, TwNatural{tw}, q, SyncCta{});
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PLAST::x_of(lt, r) * GE::C] = v[r];
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = src[(size_t)PLAST::x_of(lt, r) * GE::C];
        line_inv<GE::LOGR>(v, sm, lt, ColAddr<GE::W>{c}, TwNatural{tw}, q, SyncCta{});
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

// ---------------------------------------- fused column kernel (cluster)
// One cluster of alpha CTAs owns one (unit, column block): CTA k runs the
// inverse column pass of source limb k (input: the inverse row pass output),
// multiplies by its conversion scale and leaves the tile y_k in its shared
// memory; after a cluster barrier every CTA gathers all y tiles over
// distributed shared memory, then converts them to its share of the target
// primes (z_t = sum_k y_k c_{k,t}) and runs the forward column pass of each.
//   mode 0 (ModUp):   unit = digit j, sources q_{j alpha + k} (k < d),
//                     scale N^-1 [Dhat^-1], targets t not in D_j -> out[j][t]
//   mode 1 (ModDown): unit = half h, sources p_k (k < alpha),
//                     scale N^-1 [Phat_k^-1], targets q_i (i < l) -> out[h][i]
// grid (alpha * COL_BLOCKS, 1, units * Z), cluster (alpha, 1, 1).
namespace cgx = cooperative_groups;

// Conversion + forward column pass for targets t0 + grp, t0 + grp + NG, ...
// (NG groups of COL_THREADS threads run their targets concurrently).
template <int LOGN, int D>
__device__ __forceinline__ void colconv_targets(const Tables &T, int mode, u32 *out, size_t outz, u32 l,
                                                u32 unit, u32 z, u32 t0, u32 t1, const u32 *sy, u32 *sx,
                                                const uint2 *twt, int grp, int NG) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    const int tid = threadIdx.x % GE::COL_THREADS;
    const int c = tid % GE::W, lt = tid / GE::W;
    const int col0 = (blockIdx.x / T.alpha) * GE::W;
    const u32 ll = l + T.alpha;
    const SyncGroup gsync{1 + grp, GE::COL_THREADS};
    for (u32 ti = t0 + grp; ti < t1; ti += NG) {
        u32 g;
        const u32 *conv;
        u32 *dst;
        if (mode == 0) {
            const u32 lo = unit * T.alpha;
            const u32 t = ti < lo ? ti : ti + D;
            g = glob_of(T, l, t);
            conv = T.upConv + (((size_t)unit * T.alpha + (D - 1)) * T.NP + g) * T.alpha;
            dst = out + z * outz + ((size_t)unit * ll + t) * GE::N;
        } else {
            g = ti;
            conv = T.downConv + (size_t)ti * T.alpha;
            dst = out + z * outz + ((size_t)unit * l + ti) * GE::N;
        }
        const u32 q = T.pk[g].q, qn = T.pk[g].qn, q1s = T.pk[g].q1s;
        u32 cv[D];
#pragma unroll
        for (int k = 0; k < D; ++k) cv[k] = __ldg(conv + k);
        u32 v[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int x = PF::x_of(lt, r);
            u64 acc = 0;
#pragma unroll
            for (int k = 0; k < D; ++k) {
                if (k == 4 || k == 6) acc = fold64(acc, q, q1s);
                acc += (u64)sy[(k * GE::R + x) * GE::W + c] * cv[k];
            }
            if constexpr (D <= 4) v[r] = redc((u32)acc, red1((u32)(acc >> 32), q), q, qn);
            else v[r] = redc64(acc, q, qn, q1s);
        }
        line_fwd<GE::LOGR>(v, sx + (size_t)grp * GE::COL_TILE, lt, ColAddr<GE::W>{c},
                           TwNatural{twt + (size_t)(ti - t0) * GE::R}, q, gsync);
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PLAST::x_of(lt, r) * GE::C + col0 + c] = v[r];
    }
}

template <int LOGN>
__global__ void __launch_bounds__(1024)
k_colconv(Tables T, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz, u32 l, u32 tpc) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    cgx::cluster_group cluster = cgx::this_cluster();
    extern __shared__ __align__(16) u32 dyn[];
    constexpr int TILE = GE::R * GE::W;
    const int NG = blockDim.x / GE::COL_THREADS;     // concurrent target groups
    const int grp = threadIdx.x / GE::COL_THREADS, tid = threadIdx.x % GE::COL_THREADS;
    u32 *own = dyn;                                  // [R][W] this CTA's y tile
    u32 *sy = own + TILE;                            // [alpha][R][W] gathered tiles
    u32 *sx = sy + T.alpha * TILE;                   // [NG] padded exchange tiles
    uint2 *twi = reinterpret_cast<uint2 *>(sx + (size_t)NG * GE::COL_TILE);  // [R] inverse twiddles
    uint2 *twt = twi + GE::R;                                               // [tpc][R] forward twiddles
    const u32 rank = cluster.block_rank();
    const int c = tid % GE::W, lt = tid / GE::W;
    const int col0 = (blockIdx.x / T.alpha) * GE::W;
    const u32 units = mode == 0 ? (l + T.alpha - 1) / T.alpha : 2;
    const u32 z = blockIdx.z / units, unit = blockIdx.z % units;
    const u32 ll = l + T.alpha;
    u32 d, ntarg, gsrc;
    const u32 *s0;
    if (mode == 0) {
        d = min(T.alpha, l - unit * T.alpha);
        ntarg = ll - d;
        s0 = src + z * srcz + (size_t)unit * T.alpha * GE::N;
        gsrc = unit * T.alpha + rank;
    } else {
        d = T.alpha;
        ntarg = l;
        s0 = src + z * srcz + ((size_t)unit * ll + l) * GE::N;
        gsrc = T.L + rank;
    }
    const u32 t0 = min(rank * tpc, ntarg), t1 = min(t0 + tpc, ntarg);
    // constant tables first (overlaps the predecessor's tail)
    if (rank < d)
        for (int i = threadIdx.x; i < GE::R / 2; i += blockDim.x)
            cp_async16(twi + 2 * i, T.colI + (size_t)gsrc * GE::R + 2 * i);
    for (u32 ti = t0 + grp; ti < t1; ti += NG) {
        u32 g = ti;
        if (mode == 0) {
            const u32 lo = unit * T.alpha;
            g = glob_of(T, l, ti < lo ? ti : ti + d);
        }
        for (int i = tid; i < GE::R / 2; i += GE::COL_THREADS)
            cp_async16(twt + (size_t)(ti - t0) * GE::R + 2 * i, T.colF + (size_t)g * GE::R + 2 * i);
    }
    pdl_wait();
    pdl_trigger();
    // phase 1: inverse column pass of this CTA's source limb (group 0), times its scale
    cp_async_wait_all();
    __syncthreads();
    if (rank < d && grp == 0) {
        const u32 q = T.pk[gsrc].q;
        u32 v[16];
        const u32 *sp = s0 + (size_t)rank * GE::N + col0 + c;
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = sp[(size_t)PLAST::x_of(lt, r) * GE::C];
        line_inv<GE::LOGR>(v, sx, lt, ColAddr<GE::W>{c}, TwNatural{twi}, q, SyncGroup{1, GE::COL_THREADS});
        const uint2 sc = mode == 0 ? T.upScale[(size_t)(d - 1) * T.L + gsrc] : T.downScale[rank];
#pragma unroll
        for (int r = 0; r < 16; ++r) own[PF::x_of(lt, r) * GE::W + c] = shoup(v[r], sc.x, sc.y, q);
    }
    cp_async_wait_all();
    cluster.sync();
    // phase 2: gather every y tile of the cluster over distributed shared memory
    for (u32 k = 0; k < d; ++k) {
        const uint4 *rp = reinterpret_cast<const uint4 *>(cluster.map_shared_rank(own, k));
        uint4 *lp = reinterpret_cast<uint4 *>(sy + (size_t)k * TILE);
        for (int e = threadIdx.x; e < TILE / 4; e += blockDim.x) lp[e] = rp[e];
    }
    __syncthreads();
    // phase 3: this CTA's targets, NG at a time
    switch (d) {  // uniform over the cluster
        case 1: colconv_targets<LOGN, 1>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 2: colconv_targets<LOGN, 2>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 3: colconv_targets<LOGN, 3>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 4: colconv_targets<LOGN, 4>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 5: colconv_targets<LOGN, 5>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 6: colconv_targets<LOGN, 6>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        case 7: colconv_targets<LOGN, 7>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
        default: colconv_targets<LOGN, 8>(T, mode, out, outz, l, unit, z, t0, t1, sy, sx, twt, grp, NG); break;
    }
    cluster.sync();  // no CTA leaves while another may still read its tile
}

// ------------------------------------------------------------- inner product
// grid (ROW_BLOCKS, l+alpha, Z).  For target limb t, sum over digits j of
// ext_j[t] * (b, a)_{j,g(t)}.  FUSED: ext_j[t] = forward row pass of the
// column-pass output src[j][t] (or c1[t] for t in D_j); else ext = src.
// REGEN: a from ChaCha12 (spec v1), else from the stored key.
// PINTT: special-prime limbs get the inverse row pass before the store.
template <int LOGN, bool FUSED, bool REGEN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, 8)
k_inner(Tables T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z, u32 *acc, size_t accz,
        u32 l, KeyPack kp, int pintt) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);          // [NL][C] row twiddles
    u32 *sm = dyn + 2 * GE::NL * GE::C;                      // [NL][ROW_LS] exchange
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 t = blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    const size_t rowoff = (size_t)row * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    if (FUSED) stage_row_tw<GE>(stw, T.rowF + (size_t)g * GE::N + (size_t)row0 * GE::C);
    pdl_wait();
    pdl_trigger();
    u32 seed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) seed[i] = kp.seed[z][i];
    const u32 *kb = kp.b[z];
    const u32 *ka = kp.a[z];
    const size_t LLN = (size_t)(T.L + T.alpha) * GE::N;

    u64 sb[16], sa[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) { sb[r] = 0; sa[r] = 0; }
    bool tw_ready = !FUSED;  // uniform over the CTA

    for (u32 j = 0; j < beta; ++j) {
        const bool own = (t < l) && (t / T.alpha == j);
        // 1. issue this digit's global loads
        u32 v[16], bv[16], av[16];
        if (FUSED && !own) gload<PF>(v, src + z * srcz + ((size_t)j * ll + t) * GE::N + rowoff, lt);
        else if (FUSED) gload<PLAST>(v, c1 + z * c1z + (size_t)t * GE::N + rowoff, lt);
        else gload<PLAST>(v, src + z * srcz + ((size_t)j * ll + t) * GE::N + rowoff, lt);
        gload<PLAST>(bv, kb + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        if constexpr (!REGEN) gload<PLAST>(av, ka + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        // 2. regenerate a_{j,g} (pure ALU work, overlaps the loads above):
        //    the thread's elements form groups of KK consecutive coefficients
        if constexpr (REGEN) {
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
                        // a * 2^-32 mod q from the 64-bit word pair
                        av[gi * PLAST::KK + bb * 8 + w] = redc(ks[2 * wi], mod32(ks[2 * wi + 1], q, pk.q1s), q, pk.qn);
                    }
                }
            }
        }
        // 3. finish the NTT of the converted limb (forward row pass)
        if (FUSED && !own) {
            if (!tw_ready) {
                cp_async_wait_all();
                __syncthreads();
                tw_ready = true;
            }
            line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
        }
        // 4. multiply-accumulate; fold the 64-bit sums every two digits
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
        cp_async_wait_all();
        __syncthreads();  // every reader of the forward table is done
        stage_row_tw<GE>(stw, T.rowI + (size_t)g * GE::N + (size_t)row0 * GE::C);
        cp_async_wait_all();
        __syncthreads();
        line_inv<GE::LOGC>(ob, line, lt, RowAddr{}, tw, q, SyncWarp{});
        gstore<PF>(ob, d0, lt);
        line_inv<GE::LOGC>(oa, line, lt, RowAddr{}, tw, q, SyncWarp{});
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
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);
    u32 *sm = dyn + 2 * GE::NL * GE::C;
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 i = blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha;
    const PrimeK pk = T.pk[i];
    const u32 q = pk.q;
    const uint2 pinv = T.pInv[i];
    const size_t rowoff = (size_t)row * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    stage_row_tw<GE>(stw, T.rowF + (size_t)i * GE::N + (size_t)row0 * GE::C);
    pdl_wait();
    pdl_trigger();
    u32 v0[16], v1[16];
    gload<PF>(v0, U + z * Uz + (size_t)i * GE::N + rowoff, lt);
    gload<PF>(v1, U + z * Uz + ((size_t)l + i) * GE::N + rowoff, lt);
    cp_async_wait_all();
    __syncthreads();
    auto half = [&](u32(&v)[16], const int h) {
        u32 a[16];
        gload<PLAST>(a, acc + z * accz + ((size_t)h * ll + i) * GE::N + rowoff, lt);
        line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
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
    };
    half(v0, 0);
    half(v1, 1);
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
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);
    u32 *sm = dyn + 2 * GE::NL * GE::C;
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 t = blockIdx.y, j = blockIdx.z;
    const u32 ll = l + T.alpha;
    const u32 g = glob_of(T, l, t);
    const u32 q = T.pk[g].q;
    const size_t rowoff = (size_t)row * GE::C;
    u32 *dst = ext + ((size_t)j * ll + t) * GE::N + rowoff;
    u32 v[16];
    pdl_wait();
    pdl_trigger();
    if (t < l && t / T.alpha == j) {
        gload<PLAST>(v, c1 + (size_t)t * GE::N + rowoff, lt);
        gstore<PLAST>(v, dst, lt);
        return;
    }
    stage_row_tw<GE>(stw, T.rowF + (size_t)g * GE::N + (size_t)row0 * GE::C);
    gload<PF>(v, dst, lt);
    cp_async_wait_all();
    __syncthreads();
    line_fwd<GE::LOGC>(v, sm + rho * GE::ROW_LS, lt, RowAddr{}, TwRow{stw + rho * GE::C}, q, SyncWarp{});
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
    pdl_wait();
    pdl_trigger();
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

// Every launch goes through cudaLaunchKernelEx with programmatic stream
// serialisation (the kernels call pdl_wait before touching data) and, when the
// context has one, an L2 access-policy window that keeps the constant tables
// persisting in L2 while the streamed operands pass through.
template <typename... KArgs, typename... Args>
static cudaError_t launch_exc(const pc_ctx *c, unsigned cluster_x, void (*kern)(KArgs...), dim3 grid, dim3 block,
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
static cudaError_t launch_ex(const pc_ctx *c, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args... args) {
    return launch_exc(c, 1, kern, grid, block, smem, s, args...);
}

// targets per CTA of k_colconv, concurrent target groups, dynamic shared memory
static u32 colconv_tpc(const pc_ctx *c, int mode, u32 l) {
    const u32 ntarg_max = mode == 0 ? l + c->alpha - 1 : l;
    return (ntarg_max + c->alpha - 1) / c->alpha;
}
template <int LG>
static u32 colconv_groups(u32 tpc) {
    using GE = Geo<LG>;
    const u32 maxg = 1024 / GE::COL_THREADS;
    const u32 g = tpc < 4 ? tpc : 4;
    return g < maxg ? (g ? g : 1) : maxg;
}
template <int LG>
static size_t colconv_smem(const pc_ctx *c, u32 tpc) {
    using GE = Geo<LG>;
    return sizeof(u32) * ((size_t)(1 + c->alpha) * GE::R * GE::W + (size_t)colconv_groups<LG>(tpc) * GE::COL_TILE) +
           sizeof(uint2) * (size_t)(1 + tpc) * GE::R;
}

template <class F>
static cudaError_t allow_smem(F *f, size_t bytes) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t prepare_kernels(const pc_ctx *c) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        const size_t rs = row_smem_bytes<GE>();
        cudaError_t e = allow_smem(k_row<LG, true>, rs);
        if (e == cudaSuccess) e = allow_smem(k_row<LG, false>, rs);
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, true, true>, rs);
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, true, false>, rs);
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, false, true>, rs);
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, false, false>, rs);
        if (e == cudaSuccess) e = allow_smem(k_moddown_row<LG>, rs);
        if (e == cudaSuccess) e = allow_smem(k_modup_finish<LG>, rs);
        // the largest k_colconv instance: ModUp at the top level
        if (e == cudaSuccess) e = allow_smem(k_colconv<LG>, colconv_smem<LG>(c, colconv_tpc(c, 0, c->L)));
        if (e != cudaSuccess) return e;
    });
    return cudaSuccess;
}

cudaError_t launch_row(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime,
                       u32 nlimbs, u32 Z, size_t zin, size_t zout, bool canonical, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, nlimbs, Z);
        if (fwd) e = launch_ex(c, k_row<LG, true>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, in, out, first_prime, zin, zout, canonical);
        else e = launch_ex(c, k_row<LG, false>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, in, out, first_prime, zin, zout, canonical);
    });
    return e;
}

cudaError_t launch_col(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime,
                       u32 nlimbs, u32 Z, size_t zin, size_t zout, int scale_mode, u32 l,
                       cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::COL_BLOCKS, nlimbs, Z);
        if (fwd) e = launch_ex(c, k_col<LG, true>, grid, dim3(GE::COL_THREADS), 0, s, c->tab, in, out, first_prime, zin, zout, scale_mode, l);
        else e = launch_ex(c, k_col<LG, false>, grid, dim3(GE::COL_THREADS), 0, s, c->tab, in, out, first_prime, zin, zout, scale_mode, l);
    });
    return e;
}

cudaError_t launch_colconv(const pc_ctx *c, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz,
                           u32 l, u32 Z, cudaStream_t s) {
    const u32 units = mode == 0 ? (l + c->alpha - 1) / c->alpha : 2;
    const u32 tpc = colconv_tpc(c, mode, l);
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(c->alpha * GE::COL_BLOCKS, 1, units * Z);
        e = launch_exc(c, c->alpha, k_colconv<LG>, grid, dim3(GE::COL_THREADS * colconv_groups<LG>(tpc)),
                       colconv_smem<LG>(c, tpc), s, c->tab, mode, src, srcz, out, outz, l, tpc);
    });
    return e;
}

cudaError_t launch_inner(const pc_ctx *c, bool fused, const u32 *src, size_t srcz,
                         const u32 *c1, size_t c1z, u32 *acc, size_t accz, u32 l, const KeyPack &kp,
                         u32 Z, bool regen, bool pintt, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l + c->alpha, Z);
        if (fused && regen) e = launch_ex(c, k_inner<LG, true, true>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else if (fused) e = launch_ex(c, k_inner<LG, true, false>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else if (regen) e = launch_ex(c, k_inner<LG, false, true>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
        else e = launch_ex(c, k_inner<LG, false, false>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, src, srcz, c1, c1z, acc, accz, l, kp, pintt);
    });
    return e;
}

cudaError_t launch_moddown_row(const pc_ctx *c, const u32 *U, size_t Uz, const u32 *acc,
                               size_t accz, const u32 *c0, size_t c0z, u32 *out0, u32 *out1,
                               size_t outz, u32 l, u32 Z, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l, Z);
        e = launch_ex(c, k_moddown_row<LG>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, U, Uz, acc, accz, c0, c0z, out0, out1, outz, l);
    });
    return e;
}

cudaError_t launch_modup_finish(const pc_ctx *c, const u32 *c1, u32 *ext, u32 l, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l + c->alpha, (l + c->alpha - 1) / c->alpha);
        e = launch_ex(c, k_modup_finish<LG>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(), s, c->tab, c1, ext, l);
    });
    return e;
}

cudaError_t launch_expand(const pc_ctx *c, const u32 seed[8], u32 l, u32 *out, cudaStream_t s) {
    KeyPack kp{};
    for (int i = 0; i < 8; ++i) kp.seed[0][i] = seed[i];
    const u64 total = (u64)((l + c->alpha - 1) / c->alpha) * (l + c->alpha) * (c->N / 8);
    const u32 threads = 256;
    const u32 blocks = (u32)((total + threads - 1) / threads);
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, { e = launch_ex(c, k_expand<LG>, blocks, dim3(threads), 0, s, c->tab, kp, l, out); });
    return e;
}

}  // namespace pc
