// kernels.cu -- the key-switching kernels for sm_100a and their launchers.
//
// Dataflow of one key switch at level l (hybrid key switching, Han-Ki 2020;
// full-RNS CKKS, Cheon et al. 2018), with N = R x C viewed as R rows of C
// words.  The intermediates between a row pass and a column pass are stored
// column-major ("CM": element (r, c) at c*R + r) so that every column is
// contiguous; row kernels transpose through a shared-memory tile.
//   k_row(inv, CM out)  inverse row pass of c1                         -> W1 (CM)
//   k_colconv(ModUp)    per digit j and 2-column strip: warp k runs the
//                       inverse column pass of limb k of D_j times
//                       N^-1 [Dhat_k^-1]; the warps then convert to every
//                       target t outside D_j (z_t = sum_k y_k [Dhat_k]_t) and
//                       run its forward column pass                    -> T (CM)
//   k_inner             per target limb t and 8-row block: forward row pass
//                       of T[j][t] (or the input limb when t is in D_j), times
//                       b_{j,t} and the ChaCha12-regenerated a_{j,t}, summed
//                       over j; special-prime limbs then get the inverse row
//                       pass                                             -> ACC
//   k_colconv(ModDown)  per half and strip: inverse column pass of the
//                       special limbs times N^-1 [Phat_p^-1], conversion to
//                       every q_i, forward column pass                   -> U (CM)
//   k_moddown_row       forward row pass of U, (acc - z) [P^-1] (+ c0)   -> out
// Values between passes are lazy ([0, 2q)); every stored result of an ABI
// call is canonical.
#include <cuda_runtime.h>

#include <cstdlib>

#include <cooperative_groups.h>

#include <type_traits>

#include "chacha.cuh"
#include "ntt.cuh"
#include "launch.cuh"
#include "pc_internal.h"

namespace pc {

// Minimum resident CTAs per SM given to __launch_bounds__.  Without one,
// ptxas fits the kernels into 32 registers (full occupancy); these
// latency-bound kernels run faster with the registers they naturally use
// (48-128), which keep more independent loads and butterflies in flight.
// The conversion kernel's bound is for its largest block (8 warps): 2 CTAs
// caps it at 128 registers, so that 3 CTAs of 5 warps (alpha = 5, the
// N=2^17 basis) fit an SM -- unbounded, its N=2^17 build took 146 and 2 fit.
#ifndef PC_ROW_MIN_CTAS
#define PC_ROW_MIN_CTAS 8
#endif
#ifndef PC_COLCONV_MIN_CTAS
#define PC_COLCONV_MIN_CTAS 2
#endif
#ifndef PC_INNER_MIN_CTAS
#define PC_INNER_MIN_CTAS 4
#endif
#ifndef PC_INNER_WS_MIN_CTAS
#define PC_INNER_WS_MIN_CTAS 2
#endif
#ifndef PC_MODDOWN_MIN_CTAS
#define PC_MODDOWN_MIN_CTAS 6
#endif
constexpr int ROW_MIN_CTAS = PC_ROW_MIN_CTAS;
constexpr int COLCONV_MIN_CTAS = PC_COLCONV_MIN_CTAS;
constexpr int INNER_MIN_CTAS = PC_INNER_MIN_CTAS;
constexpr int MODDOWN_MIN_CTAS = PC_MODDOWN_MIN_CTAS;
// depth of the two-group inner product's ring of regenerated 'a' buffers and
// its named-barrier ids (FULL[s], EMPTY[s]; hardware ids go up to 15)
#ifndef PC_WS_RING
#define PC_WS_RING 6
#endif
constexpr int WS_RING = PC_WS_RING;
static_assert(WS_RING >= 2 && 2 * WS_RING + 1 <= 15, "named barrier ids 2 .. 2 WS_RING + 1");

// ------------------------------------------------------- per-CTA timeline
// Built with -DPC_TIMELINE only: each key-switching kernel stamps its CTA's
// start and end (%globaltimer, ns) and SM id, as the CTA's thread 0 exits,
// into g_tl[role][CTA index]; timeline_read copies the array out.
#ifdef PC_TIMELINE
namespace {
__device__ unsigned long long g_tl[PC_TL_ROLES][PC_TL_CTAS][3];
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
struct TlStamp {
    int role;
    unsigned long long t0;
    __device__ explicit TlStamp(int r) : role(r), t0(global_ns()) {}
    __device__ ~TlStamp() {
        if (threadIdx.x != 0) return;
        const unsigned b = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        if (b >= PC_TL_CTAS) return;
        unsigned sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        g_tl[role][b][0] = t0;
        g_tl[role][b][1] = global_ns();
        g_tl[role][b][2] = sm;
    }
};
#define PC_TL(role) const TlStamp pc_tl_stamp_(role)
#else
#define PC_TL(role) ((void)0)
#endif

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

// ------------------------------------------- automorphisms and slot products
// X -> X^g (g odd) on an NTT-domain limb is a slot permutation: slot k holds
// the value at psi^(2 brv(k) + 1), so slot k of x(X^g) is slot k' of x with
// 2 brv(k') + 1 = g (2 brv(k) + 1) mod 2N.  In the R x C view every row goes
// to a single row and every aligned block of 8 rows to an aligned block.
template <int LOGN>
__device__ __forceinline__ u32 auto_src(u32 k, u32 g) {
    const u32 idx = __brev(k) >> (32 - LOGN);
    const u32 e = (g * (2u * idx + 1u)) & ((2u << LOGN) - 1u);  // mod 2N (a power of two)
    return __brev(e >> 1) >> (32 - LOGN);
}

// a b mod q, canonical, for a, b < q: REDC of the product gives a b 2^-32.
__device__ __forceinline__ u32 mulmod(u32 a, u32 b, const PrimeK &pk) {
    const u64 p = (u64)a * b;
    return shoup(redc((u32)p, (u32)(p >> 32), pk.q, pk.qn), pk.r32, pk.r32s, pk.q);
}

// Elements x_of(lt, r) (layout PH) of row `row` of the limb x(X^g) (g = 1:
// x itself), times the same elements of y(X^g) when y is given (the slot-wise
// product of a ciphertext tensor).  Inputs canonical.
template <class PH, int LOGN, int C>
__device__ __forceinline__ void load_row_in(u32 v[16], const u32 *x, const u32 *y, int row, int lt, u32 g,
                                            const PrimeK &pk) {
    if (g == 1) {
        gload<PH>(v, x + (size_t)row * C, lt);
        if (y) {
            u32 w[16];
            gload<PH>(w, y + (size_t)row * C, lt);
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = mulmod(v[r], w[r], pk);
        }
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const u32 k = auto_src<LOGN>((u32)(row * C + PH::x_of(lt, r)), g);
            v[r] = __ldg(x + k);
            if (y) v[r] = mulmod(v[r], __ldg(y + k), pk);
        }
    }
}
// Elements x_of(lt, r) (layout PH) of row `row` of limb `limb` of half h of
// the giant-step operand W = sum_j d_j (.) bs_j (MacIn), read through
// X -> X^g: 64-bit sums of the products, folded before each product after the
// second, one reduction.  Inputs canonical; output canonical.
template <class PH, int LOGN, int C>
__device__ __forceinline__ void load_row_mac(u32 v[16], const MacIn &m, int h, u32 limb, int row, int lt, u32 g,
                                             const PrimeK &pk) {
    const size_t lo = (size_t)limb << LOGN;
    u32 k[16];
    u64 acc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const u32 x = (u32)(row * C + PH::x_of(lt, r));
        k[r] = g == 1 ? x : auto_src<LOGN>(x, g);
        acc[r] = (u64)__ldg(m.d + lo + k[r]) * __ldg(m.x0[h] + lo + k[r]);
    }
    for (u32 j = 1; j < m.n1; ++j) {
        const u32 *dj = m.d + j * m.dz + lo;
        const u32 *xj = m.xs + (j - 1) * m.xz + h * m.hz + lo;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            if (j >= 2) acc[r] = fold64(acc[r], pk.q, pk.q1s);
            acc[r] += (u64)__ldg(dj + k[r]) * __ldg(xj + k[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) v[r] = shoup(redc64(acc[r], pk.q, pk.qn, pk.q1s), pk.r32, pk.r32s, pk.q);
}

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

// Column-major staging tile of a row block (NL = 8 rows): for each of the C
// columns, the block's 8 words as two 16-byte chunks, the chunk order
// flipped on every other group of 4 columns so that a row's threads writing
// consecutive columns spread over the banks.
__device__ __forceinline__ int cm_addr(int x, int rho) {
    return x * 8 + (((rho >> 2) ^ ((x >> 2) & 1)) << 2) + (rho & 3);
}
__device__ __forceinline__ int cm_chunk(int x, int h) { return x * 8 + ((h ^ ((x >> 2) & 1)) << 2); }

// Asynchronously copy the 8 rows [row0, row0+8) of a column-major limb
// (column x at x*R) into a staging tile.  Caller commits / waits.
template <class GE>
__device__ __forceinline__ void stage_cm_rows(u32 *tile, const u32 *limb_cm, int row0) {
    static_assert(GE::NL == 8, "column-major row blocks are 8 rows (32-byte column segments)");
    constexpr int CHUNKS = 2 * GE::C;
#pragma unroll
    for (int i = 0; i < CHUNKS / GE::ROW_THREADS; ++i) {
        const int e = threadIdx.x + i * GE::ROW_THREADS;
        const int x = e >> 1, h = e & 1;
        cp_async16(tile + cm_chunk(x, h), limb_cm + (size_t)x * GE::R + row0 + 4 * h);
    }
}

// Write a staging tile (filled through cm_addr) to the 8 rows [row0, row0+8)
// of a column-major limb, 16 bytes per access.  Caller synchronises first.
template <class GE>
__device__ __forceinline__ void store_cm_rows(const u32 *tile, u32 *limb_cm, int row0) {
    constexpr int CHUNKS = 2 * GE::C;
#pragma unroll
    for (int i = 0; i < CHUNKS / GE::ROW_THREADS; ++i) {
        const int e = threadIdx.x + i * GE::ROW_THREADS;
        const int x = e >> 1, h = e & 1;
        *reinterpret_cast<uint4 *>(limb_cm + (size_t)x * GE::R + row0 + 4 * h) =
            *reinterpret_cast<const uint4 *>(tile + cm_chunk(x, h));
    }
}

// Shared memory of the row kernels: twiddles [NL][C] uint2, exchange lines
// [NL][ROW_LS], `tiles` column-major staging tiles of C*8 words.
template <class GE>
constexpr size_t row_smem_bytes(int tiles) {
    return sizeof(uint2) * GE::NL * GE::C + sizeof(u32) * (GE::NL * GE::ROW_LS + (size_t)tiles * GE::C * 8);
}

// ------------------------------------------------------------------ row pass
// grid (ROW_BLOCKS, nlimbs, Z).  Row-major limbs in.  Out: row-major (in
// place allowed), or for CMOUT (inverse only) column-major limbs.
template <int LOGN, bool FWD, bool CMOUT, bool MAC = false>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, ROW_MIN_CTAS)
k_row(Tables T, const u32 *in, u32 *out, u32 first_prime, size_t zin, size_t zout, int canonical, u32 galois,
      const u32 *mul, u32 *xout, MacIn mac) {
    PC_TL(CMOUT ? PC_TL_ROW_C1 : PC_TL_ROW_OTHER);
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    static_assert(!(CMOUT && FWD), "column-major output is for the inverse pass");
    static_assert(!(MAC && FWD), "the giant-step operand is read by the inverse pass");
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);  // [NL][C]
    u32 *sm = dyn + 2 * GE::NL * GE::C;             // [NL][ROW_LS]
    u32 *tile = sm + GE::NL * GE::ROW_LS;           // [C][8]
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 g = first_prime + blockIdx.y;
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    stage_row_tw<GE>(stw, (FWD ? T.rowF : T.rowI) + (size_t)g * GE::N + (size_t)row0 * GE::C);
    pdl_wait();
    pdl_trigger();
    const size_t limb = (size_t)blockIdx.y * GE::N;
    const u32 *src = in + blockIdx.z * zin + limb;
    u32 *dst = out + blockIdx.z * zout + limb;
    u32 v[16];
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    // the inverse pass reads a ciphertext limb, optionally through an
    // automorphism and / or times a second limb (relinearisation's d2)
    if constexpr (FWD) {
        gload<PF>(v, src + (size_t)row * GE::C, lt);
    } else {
        // (MAC: a giant step's operand, half 1, formed from the baby steps)
        if constexpr (MAC) load_row_mac<PLAST, LOGN, GE::C>(v, mac, 1, blockIdx.y, row, lt, galois, pk);
        else load_row_in<PLAST, LOGN, GE::C>(v, src, mul ? mul + blockIdx.z * zin + limb : nullptr, row, lt, galois, pk);
        // the transformed input itself (row-major, stride zout) for later readers
        if (xout) gstore<PLAST>(v, xout + blockIdx.z * zout + limb + (size_t)row * GE::C, lt);
    }
    cp_async_wait_all();
    __syncthreads();
    if constexpr (FWD) line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
    else line_inv<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
    if (canonical) {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = red1(v[r], q);
    }
    if constexpr (CMOUT) {
#pragma unroll
        for (int r = 0; r < 16; ++r) tile[cm_addr(PF::x_of(lt, r), rho)] = v[r];
        __syncthreads();
        store_cm_rows<GE>(tile, dst, row0);
    } else if constexpr (FWD) {
        gstore<PLAST>(v, dst + (size_t)row * GE::C, lt);
    } else {
        gstore<PF>(v, dst + (size_t)row * GE::C, lt);
    }
}

// -------------------------------------------- column pass, row-major limbs
// (the NTT calls).  grid (COL_BLOCKS, nlimbs, Z).  In place allowed.
// scale_mode 0: lazy output; 1: times N^-1, canonical.
template <int LOGN, bool FWD>
__global__ void __launch_bounds__(Geo<LOGN>::COL_THREADS, ROW_MIN_CTAS)
k_col(Tables T, const u32 *in, u32 *out, u32 first_prime, size_t zin, size_t zout, int scale_mode) {
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
        line_fwd<GE::LOGR>(v, sm, lt, ColAddr<GE::W>{c}, TwRow{tw}, q, SyncCta{});
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PLAST::x_of(lt, r) * GE::C] = v[r];
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = src[(size_t)PLAST::x_of(lt, r) * GE::C];
        line_inv<GE::LOGR>(v, sm, lt, ColAddr<GE::W>{c}, TwRow{tw}, q, SyncCta{});
        if (scale_mode == 1) {
            const u32 s = T.pk[g].ninv, ss = T.pk[g].ninvs;
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = shoup(v[r], s, ss, q);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[(size_t)PF::x_of(lt, r) * GE::C] = v[r];
    }
}

// ------------------------------------------------- column conversion kernel
// y tiles of the conversion kernel: each lane's 16 values of a source limb are
// stored as one run of YT_LS words (16 + 4 padding), so the targets read them
// with four 16-byte loads; lanes 20 words apart put any 8 consecutive lanes'
// 16-byte accesses on distinct bank groups.
constexpr int YT_LS = 20;

// One CTA of alpha warps per item (unit, strip of CPW columns), or per part of
// an item's targets; a column is held by TPCOL consecutive lanes, so every
// exchange is warp-synchronous.
//   mode 0 (ModUp):   unit = digit j; warp k < d runs the inverse column pass
//                     of limb q_{j alpha + k} (column-major input) times
//                     N^-1 [Dhat_k^-1]; targets t not in D_j -> out[j][t]
//   mode 1 (ModDown): unit = half h; warp k runs the inverse column pass of
//                     special limb k of ACC half h times N^-1 [Phat_k^-1];
//                     targets q_i, i < l -> out[h][i]
// The warps then share the y tiles through shared memory and take the
// targets round-robin: z_t = sum_k y_k [hat_k]_t (Montgomery constants, one
// REDC), forward column pass, store (column-major, or row-major for OUT_CM
// false).  1-D grid over the items (strip, unit, z), strip fastest, each
// item's targets in `split` parts (colconv_split); block 32 * alpha.
template <int LOGN, int D, bool OUT_CM>
__device__ __forceinline__ void colconv_targets(const Tables &T, int mode, u32 *out, size_t outz, u32 l, u32 unit,
                                                u32 z, u32 tlo, u32 thi, const u32 *sy, u32 *xl0, int c, int lt,
                                                int col) {
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    const u32 ll = l + T.alpha;
    const u32 warp = threadIdx.x / 32, nwarps = blockDim.x / 32;
    // target ti -> (prime, conversion constants, output limb)
    auto target = [&](u32 ti, u32 &g, const u32 *&conv, u32 *&dst) {
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
    };
    // one target per warp at a time (a short loop body: the kernel is
    // latency-bound and a two-target body overflowed the instruction cache)
    for (u32 ti = tlo + warp; ti < thi; ti += nwarps) {
        u32 g0;
        const u32 *conv0;
        u32 *dst0;
        target(ti, g0, conv0, dst0);
        const u32 q0 = T.pk[g0].q, qn0 = T.pk[g0].qn, q1s0 = T.pk[g0].q1s;
        u32 cv0[D];
#pragma unroll
        for (int k = 0; k < D; ++k) cv0[k] = __ldg(conv0 + k);
        u32 v0[16];
        // the lane's 16 values of source k are one contiguous run (see YT_LS)
        const u32 *yl = sy + (c * GE::TPCOL + lt) * YT_LS;
#pragma unroll
        for (int rc = 0; rc < 4; ++rc) {
            u64 a0[4] = {0, 0, 0, 0};
#pragma unroll
            for (int k = 0; k < D; ++k) {
                const uint4 y4 = *reinterpret_cast<const uint4 *>(yl + k * GE::CPW * GE::TPCOL * YT_LS + 4 * rc);
                const u32 yv[4] = {y4.x, y4.y, y4.z, y4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (k == 4 || k == 6) a0[i] = fold64(a0[i], q0, q1s0);
                    a0[i] += (u64)yv[i] * cv0[k];
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (D <= 4) v0[4 * rc + i] = redc((u32)a0[i], red1((u32)(a0[i] >> 32), q0), q0, qn0);
                else v0[4 * rc + i] = redc64(a0[i], q0, qn0, q1s0);
            }
        }
        line_fwd<GE::LOGR>(v0, xl0, lt, Pad4Addr{}, TwRowG{T.colF + (size_t)g0 * GE::R}, q0, SyncWarp{});
        if constexpr (OUT_CM) {
            gstore<PLAST>(v0, dst0 + (size_t)col * GE::R, lt);
        } else {
#pragma unroll
            for (int r = 0; r < 16; ++r) dst0[(size_t)PLAST::x_of(lt, r) * GE::C + col] = v0[r];
        }
    }
}

template <int LOGN, bool OUT_CM>
__global__ void __launch_bounds__(32 * MAX_ALPHA, COLCONV_MIN_CTAS)
k_colconv(Tables T, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz, u32 l, u32 split) {
    PC_TL(mode == 0 ? PC_TL_CONV_UP : PC_TL_CONV_DOWN);
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGR>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGR>::type;
    extern __shared__ __align__(16) u32 dyn[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int c = lane / GE::TPCOL, lt = lane % GE::TPCOL;
    // item (strip, unit, z) and the part of its targets this CTA converts
    constexpr u32 STRIPS = GE::C / GE::CPW;
    const u32 item = blockIdx.x / split, part = blockIdx.x % split;
    const int col = (int)(item % STRIPS) * GE::CPW + c;
    u32 *sy = dyn;                                          // [alpha][CPW][TPCOL][YT_LS] y tiles
    // one exchange line per warp and column, after the y tiles
    u32 *xl = dyn + T.alpha * GE::CPW * GE::TPCOL * YT_LS + (warp * GE::CPW + c) * GE::COL_LS4;
    const u32 units = mode == 0 ? (l + T.alpha - 1) / T.alpha : 2;
    const u32 z = item / STRIPS / units, unit = item / STRIPS % units;
    const u32 ll = l + T.alpha;
    u32 d, ntarg, gsrc;
    const u32 *s0;
    if (mode == 0) {
        d = min(T.alpha, l - unit * T.alpha);
        ntarg = ll - d;
        s0 = src + z * srcz + (size_t)unit * T.alpha * GE::N;
        gsrc = unit * T.alpha + warp;
    } else {
        d = T.alpha;
        ntarg = l;
        s0 = src + z * srcz + ((size_t)unit * ll + l) * GE::N;
        gsrc = T.L + warp;
    }
    pdl_wait();
    pdl_trigger();
    if ((u32)warp < d) {
        const u32 q = T.pk[gsrc].q;
        u32 v[16];
        gload<PLAST>(v, s0 + (size_t)warp * GE::N + (size_t)col * GE::R, lt);
        line_inv<GE::LOGR>(v, xl, lt, Pad4Addr{}, TwRowG{T.colI + (size_t)gsrc * GE::R}, q, SyncWarp{});
        const uint2 sc = mode == 0 ? T.upScale[(size_t)(d - 1) * T.L + gsrc] : T.downScale[warp];
        // the lane's 16 values (PF positions lt + TPCOL r) as one contiguous run
        u32 *yt = sy + ((warp * GE::CPW + c) * GE::TPCOL + lt) * YT_LS;
#pragma unroll
        for (int r = 0; r < 16; r += 4)
            *reinterpret_cast<uint4 *>(yt + r) = make_uint4(shoup(v[r], sc.x, sc.y, q), shoup(v[r + 1], sc.x, sc.y, q),
                                                            shoup(v[r + 2], sc.x, sc.y, q), shoup(v[r + 3], sc.x, sc.y, q));
    }
    __syncthreads();
    const u32 tlo = ntarg * part / split, thi = ntarg * (part + 1) / split;
    switch (d) {  // uniform over the CTA
        case 1: colconv_targets<LOGN, 1, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 2: colconv_targets<LOGN, 2, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 3: colconv_targets<LOGN, 3, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 4: colconv_targets<LOGN, 4, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 5: colconv_targets<LOGN, 5, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 6: colconv_targets<LOGN, 6, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        case 7: colconv_targets<LOGN, 7, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
        default: colconv_targets<LOGN, 8, OUT_CM>(T, mode, out, outz, l, unit, z, tlo, thi, sy, xl, c, lt, col); break;
    }
}

// ------------------------------------------------------------- inner product
// grid (ROW_BLOCKS, nt, Z), target limb t = t0 + blockIdx.y.  Sum over digits j of
// ext_j[t] * (b, a)_{j,g(t)}.  FUSED: ext_j[t] = forward row pass of the
// column-major column-pass output src[j][t] (or c1[t] for t in D_j), staged
// through shared memory one digit ahead; else ext = src (row-major).
// REGEN: a from ChaCha12 (spec v1), else from the stored key.
// PINTT: special-prime limbs get the inverse row pass and are stored
// column-major (the ModDown column kernel reads them so).
// k_inner_rot (hoisted rotation, fused): ext_j is replaced by
// ext_j(X^galois).  Each thread-row loads a source row of the block that the
// automorphism maps onto this CTA's output rows (for a converted limb it runs
// the row pass on it), then permutes the row's columns through shared memory
// into its output row; ginv = galois^-1 mod 2N.  Its body, inner_body, also
// covers ROT = false, but k_inner keeps a text of its own: instantiated from
// the shared body, ptxas scheduled the plain kernel's loads later (twice the
// long-scoreboard stalls at the same instruction count; 84 instead of 80 us
// at N=2^16, l=24).
enum { XF_PLAIN = 0, XF_GATHER = 1, XF_MUL = 3, XF_MAC = 4 };  // input modes of the ModDown finish
template <int LOGN, bool FUSED, bool REGEN, bool ROT>
__device__ __forceinline__ void inner_body(const Tables &T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z,
                                           u32 *acc, size_t accz, u32 l, const KeyPack &kp, int pintt, u32 t0,
                                           u32 galois, u32 ginv) {
    static_assert(FUSED || !ROT, "rotation of the extended limbs needs the fused row pass");
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);           // [NL][C] row twiddles
    u32 *sm = dyn + 2 * GE::NL * GE::C;                      // [NL][ROW_LS] exchange
    u32 *tiles = sm + GE::NL * GE::ROW_LS;                   // [2][C*8] staging
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL;
    const u32 t = t0 + blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    // thread-row rho runs the row pass of source row srow0 + rho and
    // accumulates output row orow (the same row unless ROT)
    int srow0 = row0, orow = row0 + rho;
    // ROT: source column of each of the thread's output elements, 8 bits each,
    // after the staging tiles in dynamic shared memory
    u32 *scol = tiles + 2 * GE::C * 8;
    if constexpr (ROT) {
        static_assert(GE::C <= 256, "source columns are packed in bytes");
        srow0 = (int)(auto_src<LOGN>((u32)row0 * GE::C, galois) / GE::C) & ~(GE::NL - 1);
        orow = (int)(auto_src<LOGN>((u32)(srow0 + rho) * GE::C, ginv) / GE::C);
        u32 cs[4] = {0, 0, 0, 0};
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const u32 k = auto_src<LOGN>((u32)(orow * GE::C + PLAST::x_of(lt, r)), galois);
            cs[r >> 2] |= (k & (GE::C - 1)) << (8 * (r & 3));
        }
        *reinterpret_cast<uint4 *>(scol + 4 * threadIdx.x) = make_uint4(cs[0], cs[1], cs[2], cs[3]);
    }
    const size_t rowoff = (size_t)orow * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    const u32 jown = t < l ? t / T.alpha : beta;  // the digit holding t, if any
    if (FUSED) stage_row_tw<GE>(stw, T.rowF + (size_t)g * GE::N + (size_t)srow0 * GE::C);
    // counter-free quarter rounds of every digit's ChaCha12 blocks, once per CTA
    __shared__ __align__(16) u32 spre[12 * MAX_L];
    if (REGEN && threadIdx.x < beta) {
        u32 sd[8], pre[12];
#pragma unroll
        for (int i = 0; i < 8; ++i) sd[i] = kp.seed[z][i];
        chacha12_precolumn(sd, g, threadIdx.x, pre);
#pragma unroll
        for (int i = 0; i < 12; ++i) spre[12 * threadIdx.x + i] = pre[i];
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const u32 *srcz_p = src + z * srcz;
    u32 jn = (jown == 0) ? 1 : 0;  // next converted digit to stage
    int buf = 0;
    if (FUSED && jn < beta) stage_cm_rows<GE>(tiles, srcz_p + ((size_t)jn * ll + t) * GE::N, srow0);
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
        const bool own = j == jown;
        u32 v[16], bv[16], av[16];
        if (FUSED && !own) {
            // this digit's tile has landed for every thread; the other tile's
            // readers (previous converted digit) are done: prefetch the next
            cp_async_wait_all();
            __syncthreads();
            jn = j + 1 + ((j + 1) == jown ? 1 : 0);
            if (jn < beta)
                stage_cm_rows<GE>(tiles + (buf ^ 1) * GE::C * 8, srcz_p + ((size_t)jn * ll + t) * GE::N, srow0);
            const u32 *tl = tiles + buf * GE::C * 8;
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = tl[cm_addr(PF::x_of(lt, r), rho)];
            buf ^= 1;
        } else if (FUSED) {
            // own digit: the input limb itself (ROT: its source row, permuted below)
            gload<PLAST>(v, c1 + z * c1z + (size_t)t * GE::N + (size_t)(ROT ? srow0 + rho : orow) * GE::C, lt);
        } else {
            gload<PLAST>(v, srcz_p + ((size_t)j * ll + t) * GE::N + rowoff, lt);
        }
        gload<PLAST>(bv, kb + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        if constexpr (!REGEN) gload<PLAST>(av, ka + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        // regenerate a_{j,g} (pure ALU work, overlaps the loads above): the
        // thread's elements form groups of KK consecutive coefficients
        if constexpr (REGEN && PLAST::KK == 16) {
            // the thread's 16 consecutive coefficients are two whole blocks
            const u32 base = (u32)(rowoff + PLAST::x_of(lt, 0));
            u32 o0[16], o1[16];
            u32 pre[12];
            const uint4 *pp = reinterpret_cast<const uint4 *>(spre + 12 * j);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const uint4 w4 = pp[i];
                pre[4 * i] = w4.x; pre[4 * i + 1] = w4.y; pre[4 * i + 2] = w4.z; pre[4 * i + 3] = w4.w;
            }
            chacha12_block2_pre(pre, seed, base >> 3, g, j, o0, o1);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                av[w] = redc(o0[2 * w], mod32(o0[2 * w + 1], q, pk.q1s), q, pk.qn);
                av[8 + w] = redc(o1[2 * w], mod32(o1[2 * w + 1], q, pk.q1s), q, pk.qn);
            }
        } else if constexpr (REGEN) {
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
        if (FUSED && !own) line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
        if constexpr (ROT) {
            // column x of output row orow is column colsrc of the source row
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 16; ++r) line[RowAddr{}(PLAST::x_of(lt, r))] = v[r];
            __syncwarp();
            const uint4 c4 = *reinterpret_cast<const uint4 *>(scol + 4 * threadIdx.x);
            const u32 colsrc[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = line[RowAddr{}((int)((colsrc[r >> 2] >> (8 * (r & 3))) & 0xffu))];
            __syncwarp();
        }
        // multiply-accumulate; fold the 64-bit sums every two digits
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
    u32 *d0 = acc + z * accz + (size_t)t * GE::N;
    u32 *d1 = acc + z * accz + (size_t)(ll + t) * GE::N;
    if (pintt && t >= l) {
        cp_async_wait_all();
        __syncthreads();  // every reader of the forward table and the tiles is done
        stage_row_tw<GE>(stw, T.rowI + (size_t)g * GE::N + (size_t)row0 * GE::C);
        cp_async_wait_all();
        __syncthreads();
        const TwRow twi{stw + (orow - row0) * GE::C};  // twiddles of the output row
        line_inv<GE::LOGC>(ob, line, lt, RowAddr{}, twi, q, SyncWarp{});
        line_inv<GE::LOGC>(oa, line, lt, RowAddr{}, twi, q, SyncWarp{});
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int a = cm_addr(PF::x_of(lt, r), orow - row0);
            tiles[a] = ob[r];
            tiles[GE::C * 8 + a] = oa[r];
        }
        __syncthreads();
        store_cm_rows<GE>(tiles, d0, row0);
        store_cm_rows<GE>(tiles + GE::C * 8, d1, row0);
    } else {
        gstore<PLAST>(ob, d0 + rowoff, lt);
        gstore<PLAST>(oa, d1 + rowoff, lt);
    }
}

template <int LOGN, bool FUSED, bool REGEN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, INNER_MIN_CTAS)
k_inner(Tables T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z, u32 *acc, size_t accz,
        u32 l, KeyPack kp, int pintt, u32 t0) {
    PC_TL(PC_TL_INNER_OTHER);
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);           // [NL][C] row twiddles
    u32 *sm = dyn + 2 * GE::NL * GE::C;                      // [NL][ROW_LS] exchange
    u32 *tiles = sm + GE::NL * GE::ROW_LS;                   // [2][C*8] staging
    const int rho = threadIdx.x / GE::TPR, lt = threadIdx.x % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 t = t0 + blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    const size_t rowoff = (size_t)row * GE::C;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    const u32 jown = t < l ? t / T.alpha : beta;  // the digit holding t, if any
    if (FUSED) stage_row_tw<GE>(stw, T.rowF + (size_t)g * GE::N + (size_t)row0 * GE::C);
    // counter-free quarter rounds of every digit's ChaCha12 blocks, once per CTA
    __shared__ __align__(16) u32 spre[12 * MAX_L];
    if (REGEN && threadIdx.x < beta) {
        u32 sd[8], pre[12];
#pragma unroll
        for (int i = 0; i < 8; ++i) sd[i] = kp.seed[z][i];
        chacha12_precolumn(sd, g, threadIdx.x, pre);
#pragma unroll
        for (int i = 0; i < 12; ++i) spre[12 * threadIdx.x + i] = pre[i];
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const u32 *srcz_p = src + z * srcz;
    u32 jn = (jown == 0) ? 1 : 0;  // next converted digit to stage
    int buf = 0;
    if (FUSED && jn < beta) stage_cm_rows<GE>(tiles, srcz_p + ((size_t)jn * ll + t) * GE::N, row0);
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
        const bool own = j == jown;
        u32 v[16], bv[16], av[16];
        if (FUSED && !own) {
            // this digit's tile has landed for every thread; the other tile's
            // readers (previous converted digit) are done: prefetch the next
            cp_async_wait_all();
            __syncthreads();
            jn = j + 1 + ((j + 1) == jown ? 1 : 0);
            if (jn < beta) stage_cm_rows<GE>(tiles + (buf ^ 1) * GE::C * 8, srcz_p + ((size_t)jn * ll + t) * GE::N, row0);
            const u32 *tl = tiles + buf * GE::C * 8;
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = tl[cm_addr(PF::x_of(lt, r), rho)];
            buf ^= 1;
        } else if (FUSED) {
            gload<PLAST>(v, c1 + z * c1z + (size_t)t * GE::N + rowoff, lt);
        } else {
            gload<PLAST>(v, srcz_p + ((size_t)j * ll + t) * GE::N + rowoff, lt);
        }
        gload<PLAST>(bv, kb + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        if constexpr (!REGEN) gload<PLAST>(av, ka + (size_t)j * LLN + (size_t)g * GE::N + rowoff, lt);
        // regenerate a_{j,g} (pure ALU work, overlaps the loads above): the
        // thread's elements form groups of KK consecutive coefficients
        if constexpr (REGEN && PLAST::KK == 16) {
            // the thread's 16 consecutive coefficients are two whole blocks
            const u32 base = (u32)(rowoff + PLAST::x_of(lt, 0));
            u32 o0[16], o1[16];
            u32 pre[12];
            const uint4 *pp = reinterpret_cast<const uint4 *>(spre + 12 * j);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const uint4 w4 = pp[i];
                pre[4 * i] = w4.x; pre[4 * i + 1] = w4.y; pre[4 * i + 2] = w4.z; pre[4 * i + 3] = w4.w;
            }
            chacha12_block2_pre(pre, seed, base >> 3, g, j, o0, o1);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                av[w] = redc(o0[2 * w], mod32(o0[2 * w + 1], q, pk.q1s), q, pk.qn);
                av[8 + w] = redc(o1[2 * w], mod32(o1[2 * w + 1], q, pk.q1s), q, pk.qn);
            }
        } else if constexpr (REGEN) {
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
        if (FUSED && !own) line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
        // multiply-accumulate; fold the 64-bit sums every two digits
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
    u32 *d0 = acc + z * accz + (size_t)t * GE::N;
    u32 *d1 = acc + z * accz + (size_t)(ll + t) * GE::N;
    if (pintt && t >= l) {
        cp_async_wait_all();
        __syncthreads();  // every reader of the forward table and the tiles is done
        stage_row_tw<GE>(stw, T.rowI + (size_t)g * GE::N + (size_t)row0 * GE::C);
        cp_async_wait_all();
        __syncthreads();
        line_inv<GE::LOGC>(ob, line, lt, RowAddr{}, tw, q, SyncWarp{});
        line_inv<GE::LOGC>(oa, line, lt, RowAddr{}, tw, q, SyncWarp{});
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int a = cm_addr(PF::x_of(lt, r), rho);
            tiles[a] = ob[r];
            tiles[GE::C * 8 + a] = oa[r];
        }
        __syncthreads();
        store_cm_rows<GE>(tiles, d0, row0);
        store_cm_rows<GE>(tiles + GE::C * 8, d1, row0);
    } else {
        gstore<PLAST>(ob, d0 + rowoff, lt);
        gstore<PLAST>(oa, d1 + rowoff, lt);
    }
}

// ------------------------------------- inner product, warp-specialised
// The fused inner product with regenerated 'a' (k_inner<FUSED, REGEN>'s
// result) by two groups of NT = ROW_THREADS threads each.  Group 1 (the
// producer) regenerates a_{j,g} with ChaCha12 for the CTA's rows, digit after
// digit, into a double buffer in shared memory; it reads no data written by an
// earlier kernel, so it starts while that kernel drains.  Group 0 (the
// consumer) stages the column-pass tiles and the key's 'b' half one digit
// ahead with asynchronous copies, runs the forward row passes and
// multiply-accumulates both halves.  So the ALU-bound cipher and the
// multiply-bound transforms run in different warps and overlap on the SM.
// The 'a' words pass through a ring of WS_RING buffers: the producer runs up to
// WS_RING digits ahead -- all of them at N=2^16, l=24 -- which it does while
// the consumer waits for the conversion kernel to finish.
// Hand-off: named barriers FULL[s] (ids 2 .. WS_RING + 1: the producer
// arrives once digit j's words are in buffer s = j mod WS_RING, the consumer
// waits) and EMPTY[s] (ids WS_RING + 2 .. 2 WS_RING + 1: the consumer arrives
// once it has read buffer s, if digit j + WS_RING exists; the producer waits
// before refilling it); id 1 orders the consumer group alone.  Every thread
// of a group takes the same barrier steps (beta and the own digit are uniform
// over the CTA), so each barrier phase completes.
template <int LOGN>
__global__ void __launch_bounds__(2 * Geo<LOGN>::ROW_THREADS, PC_INNER_WS_MIN_CTAS)
k_inner_ws(Tables T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z, u32 *acc, size_t accz, u32 l,
           KeyPack kp, int pintt, u32 t0) {
    PC_TL(t0 > 0 ? PC_TL_INNER_SPECIAL : PC_TL_INNER_CT);
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    static_assert(PLAST::KK == 16, "a thread's 16 coefficients are two whole ChaCha blocks");
    constexpr int NT = GE::ROW_THREADS;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);           // [NL][C] row twiddles
    u32 *sm = dyn + 2 * GE::NL * GE::C;                      // [NL][ROW_LS] exchange
    u32 *tiles = sm + GE::NL * GE::ROW_LS;                   // [2][C*8] column-pass tiles
    uint4 *bbuf = reinterpret_cast<uint4 *>(tiles + 2 * GE::C * 8);  // [2][4][NT] key 'b' words
    u32 *abuf = tiles + 2 * GE::C * 8 + 2 * 16 * NT;          // [WS_RING][16][NT] regenerated 'a'
    u32 *spre = abuf + WS_RING * 16 * NT;                      // [beta][12] first-round words
    constexpr int WS_FULL = 2, WS_EMPTY = 2 + WS_RING;  // FULL[s], EMPTY[s] barrier ids
    const bool producer = threadIdx.x >= NT;
    const int tid = producer ? threadIdx.x - NT : threadIdx.x;
    const int rho = tid / GE::TPR, lt = tid % GE::TPR;
    const int row0 = blockIdx.x * GE::NL, row = row0 + rho;
    const u32 t = t0 + blockIdx.y, z = blockIdx.z;
    const u32 ll = l + T.alpha, beta = (l + T.alpha - 1) / T.alpha;
    const u32 g = glob_of(T, l, t);
    const PrimeK pk = T.pk[g];
    const u32 q = pk.q;
    const size_t rowoff = (size_t)row * GE::C;
    const u32 jown = t < l ? t / T.alpha : beta;  // the digit holding t, if any
    // set-up: the consumer stages this CTA's forward row twiddles; producer
    // threads compute the counter-free quarter rounds of every digit's blocks
    if (!producer) stage_row_tw<GE>(stw, T.rowF + (size_t)g * GE::N + (size_t)row0 * GE::C);
    if (producer && (u32)tid < beta) {
        u32 sd[8], pre[12];
#pragma unroll
        for (int i = 0; i < 8; ++i) sd[i] = kp.seed[z][i];
        chacha12_precolumn(sd, g, tid, pre);
#pragma unroll
        for (int i = 0; i < 12; ++i) spre[12 * tid + i] = pre[i];
    }
    __syncthreads();
    if (producer) {
        pdl_trigger();
        u32 seed[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) seed[i] = kp.seed[z][i];
        const u32 base = (u32)(rowoff + PLAST::x_of(lt, 0));
        for (u32 j = 0, s = 0; j < beta; ++j, s = s + 1 == WS_RING ? 0 : s + 1) {
            if (j >= (u32)WS_RING) bar_sync(WS_EMPTY + s, 2 * NT);
            u32 o0[16], o1[16], pre[12];
            const uint4 *pp = reinterpret_cast<const uint4 *>(spre + 12 * j);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                const uint4 w4 = pp[i];
                pre[4 * i] = w4.x; pre[4 * i + 1] = w4.y; pre[4 * i + 2] = w4.z; pre[4 * i + 3] = w4.w;
            }
            chacha12_block2_pre(pre, seed, base >> 3, g, j, o0, o1);
            u32 *ab = abuf + s * 16 * NT + tid;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                // a * 2^-32 mod q from the 64-bit word pair
                ab[w * NT] = redc(o0[2 * w], mod32(o0[2 * w + 1], q, pk.q1s), q, pk.qn);
                ab[(8 + w) * NT] = redc(o1[2 * w], mod32(o1[2 * w + 1], q, pk.q1s), q, pk.qn);
            }
            bar_arrive(WS_FULL + s, 2 * NT);
        }
        return;
    }
    pdl_wait();
    pdl_trigger();
    const u32 *srcz_p = src + z * srcz;
    const u32 *kb = kp.b[z] + (size_t)g * GE::N + rowoff + PLAST::x_of(lt, 0);
    const size_t LLN = (size_t)(T.L + T.alpha) * GE::N;
    u32 *line = sm + rho * GE::ROW_LS;
    const TwRow tw{stw + rho * GE::C};
    const u32 nconv = beta - (jown < beta ? 1u : 0u);
    auto conv_digit = [&](u32 k) { return k < jown ? k : k + 1; };  // k-th converted digit
    auto stage_b = [&](u32 j) {
        const uint4 *gb = reinterpret_cast<const uint4 *>(kb + (size_t)j * LLN);
        uint4 *sb = bbuf + (j & 1) * 4 * NT + tid;
#pragma unroll
        for (int c = 0; c < 4; ++c) cp_async16(sb + c * NT, gb + c);
    };
    if (nconv) stage_cm_rows<GE>(tiles, srcz_p + ((size_t)conv_digit(0) * ll + t) * GE::N, row0);
    stage_b(0);
    cp_async_commit();

    u64 sb[16], sa[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) { sb[r] = 0; sa[r] = 0; }
    u32 kc = 0;
    for (u32 j = 0; j < beta; ++j) {
        const bool own = j == jown;
        // digit j's tile and b words have landed; the buffers refilled below
        // are no longer read by any consumer thread
        cp_async_wait_all();
        bar_sync(1, NT);
        if (j + 1 < beta) stage_b(j + 1);
        if (!own && kc + 1 < nconv)
            stage_cm_rows<GE>(tiles + ((kc + 1) & 1) * GE::C * 8,
                              srcz_p + ((size_t)conv_digit(kc + 1) * ll + t) * GE::N, row0);
        cp_async_commit();
        u32 v[16], bv[16], av[16];
        if (own) {
            gload<PLAST>(v, c1 + z * c1z + (size_t)t * GE::N + rowoff, lt);
        } else {
            const u32 *tl = tiles + (kc & 1) * GE::C * 8;
#pragma unroll
            for (int r = 0; r < 16; ++r) v[r] = tl[cm_addr(PF::x_of(lt, r), rho)];
            line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
            ++kc;
        }
        const uint4 *bb = bbuf + (j & 1) * 4 * NT + tid;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w4 = bb[c * NT];
            bv[4 * c] = w4.x; bv[4 * c + 1] = w4.y; bv[4 * c + 2] = w4.z; bv[4 * c + 3] = w4.w;
        }
        const u32 slot = j % WS_RING;
        bar_sync(WS_FULL + slot, 2 * NT);  // digit j's 'a' words are in
        const u32 *ab = abuf + slot * 16 * NT + tid;
#pragma unroll
        for (int r = 0; r < 16; ++r) av[r] = ab[r * NT];
        if (j + WS_RING < beta) bar_arrive(WS_EMPTY + slot, 2 * NT);
        // multiply-accumulate; fold the 64-bit sums every two digits
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
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        ob[r] = shoup(redc64(sb[r], q, pk.qn, pk.q1s), pk.r32, pk.r32s, q);
        oa[r] = shoup(redc64(sa[r], q, pk.qn, pk.q1s), pk.r64, pk.r64s, q);
    }
    u32 *d0 = acc + z * accz + (size_t)t * GE::N;
    u32 *d1 = acc + z * accz + (size_t)(ll + t) * GE::N;
    if (pintt && t >= l) {
        cp_async_wait_all();
        bar_sync(1, NT);  // every reader of the forward table and the tiles is done
        stage_row_tw<GE>(stw, T.rowI + (size_t)g * GE::N + (size_t)row0 * GE::C);
        cp_async_wait_all();
        bar_sync(1, NT);
        line_inv<GE::LOGC>(ob, line, lt, RowAddr{}, tw, q, SyncWarp{});
        line_inv<GE::LOGC>(oa, line, lt, RowAddr{}, tw, q, SyncWarp{});
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int a = cm_addr(PF::x_of(lt, r), rho);
            tiles[a] = ob[r];
            tiles[GE::C * 8 + a] = oa[r];
        }
        bar_sync(1, NT);
        store_cm_rows<GE>(tiles, d0, row0);
        store_cm_rows<GE>(tiles + GE::C * 8, d1, row0);
    } else {
        gstore<PLAST>(ob, d0 + rowoff, lt);
        gstore<PLAST>(oa, d1 + rowoff, lt);
    }
}

// element z of a parameter array without copying the array to local memory
__device__ __forceinline__ u32 pick(const u32 (&a)[KEYS_PER_LAUNCH], u32 z) {
    u32 v = a[0];
#pragma unroll
    for (int i = 1; i < KEYS_PER_LAUNCH; ++i) v = (z == (u32)i) ? a[i] : v;
    return v;
}

template <int LOGN, bool REGEN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, INNER_MIN_CTAS)
k_inner_rot(Tables T, const u32 *src, size_t srcz, const u32 *c1, size_t c1z, u32 *acc, size_t accz, u32 l,
            KeyPack kp, int pintt, u32 t0, RotPack rp) {
    PC_TL(PC_TL_INNER_OTHER);
    inner_body<LOGN, true, REGEN, true>(T, src, srcz, c1, c1z, acc, accz, l, kp, pintt, t0,
                                        pick(rp.galois, blockIdx.z), pick(rp.ginv, blockIdx.z));
}

// ----------------------------------------------------------- ModDown finish
// grid (ROW_BLOCKS, l, Z).  out_h[i] = (acc_h[i] - rowfwd(U_h[i])) [P^-1]_{q_i},
// plus c0 for h = 0 when c0 is given, or plus the tensor terms d0 (h = 0)
// and d1 (h = 1) of ciphertexts rx, ry ([2][l][N], Z = 1) when rx is given;
// U column-major, the rest row-major.  out0/out1 may alias c0 only for
// XF_PLAIN.
// XF: XF_PLAIN, XF_GATHER (c0 of slice z read through X -> X^rp.galois[z]),
// XF_MUL (the tensor terms of rx, ry added instead of c0) or XF_MAC (Z = 1:
// half 0 of the giant-step operand of mac, read through X -> X^rp.galois[0],
// added instead of c0, and both results added to out0 / out1 in place).
template <int LOGN, int XF>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, MODDOWN_MIN_CTAS)
k_moddown_row(Tables T, const u32 *U, size_t Uz, const u32 *acc, size_t accz, const u32 *c0,
              size_t c0z, u32 *out0, u32 *out1, size_t outz, u32 l, RotPack rp, const u32 *rx, const u32 *ry,
              MacIn mac) {
    PC_TL(PC_TL_MODDOWN_FINISH);
    using GE = Geo<LOGN>;
    using PL = Plan<GE::LOGC>;
    using PF = typename PL::P0;
    using PLAST = typename LastPhase<GE::LOGC>::type;
    extern __shared__ __align__(16) u32 dyn[];
    uint2 *stw = reinterpret_cast<uint2 *>(dyn);
    u32 *sm = dyn + 2 * GE::NL * GE::C;
    u32 *tiles = sm + GE::NL * GE::ROW_LS;
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
    // c0 is the caller's input, which no kernel of the call writes: its row
    // loads before the wait for the inner products and the ModDown conversion
    u32 ah[2][16], c0v[16];
    if constexpr (XF == XF_PLAIN) {
        if (c0) gload<PLAST>(c0v, c0 + z * c0z + (size_t)i * GE::N + rowoff, lt);
    }
    pdl_wait();
    pdl_trigger();
    stage_cm_rows<GE>(tiles, U + z * Uz + (size_t)i * GE::N, row0);
    stage_cm_rows<GE>(tiles + GE::C * 8, U + z * Uz + ((size_t)l + i) * GE::N, row0);
    // both halves' accumulator rows load while the tiles stage
    gload<PLAST>(ah[0], acc + z * accz + (size_t)i * GE::N + rowoff, lt);
    gload<PLAST>(ah[1], acc + z * accz + ((size_t)ll + i) * GE::N + rowoff, lt);
    cp_async_wait_all();
    __syncthreads();
    auto half = [&](const int h) {
        u32 v[16];
        const u32 *a = ah[h];
        const u32 *tl = tiles + h * GE::C * 8;
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = tl[cm_addr(PF::x_of(lt, r), rho)];
        line_fwd<GE::LOGC>(v, line, lt, RowAddr{}, tw, q, SyncWarp{});
        u32 o[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) o[r] = shoup(a[r] - red1(v[r], q) + q, pinv.x, pinv.y, q);
        if constexpr (XF == XF_MUL) {
            // relinearisation: + d0 = x0 y0 (h = 0), + d1 = x0 y1 + x1 y0 (h = 1)
            const size_t lN = (size_t)l * GE::N, li = (size_t)i * GE::N + rowoff;
            u32 x0[16], y0[16], cc[16];
            gload<PLAST>(x0, rx + li, lt);
            gload<PLAST>(y0, ry + li, lt);
            if (h == 0) {
#pragma unroll
                for (int r = 0; r < 16; ++r) cc[r] = mulmod(x0[r], y0[r], pk);
            } else {
                u32 x1[16], y1[16];
                gload<PLAST>(x1, rx + lN + li, lt);
                gload<PLAST>(y1, ry + lN + li, lt);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const u64 d = (u64)x0[r] * y1[r] + (u64)x1[r] * y0[r];
                    cc[r] = shoup(redc64(d, q, pk.qn, pk.q1s), pk.r32, pk.r32s, q);
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) o[r] = red1(o[r] + cc[r], q);
        } else if constexpr (XF == XF_MAC) {
            u32 cc[16];
            if (h == 0) {
                load_row_mac<PLAST, LOGN, GE::C>(cc, mac, 0, i, row, lt, rp.galois[0], pk);
#pragma unroll
                for (int r = 0; r < 16; ++r) o[r] = red1(o[r] + cc[r], q);
            }
            gload<PLAST>(cc, (h == 0 ? out0 : out1) + (size_t)i * GE::N + rowoff, lt);
#pragma unroll
            for (int r = 0; r < 16; ++r) o[r] = red1(o[r] + cc[r], q);
        } else if (h == 0 && c0) {
            u32 cc[16];
            if constexpr (XF == XF_GATHER)
                load_row_in<PLAST, LOGN, GE::C>(cc, c0 + z * c0z + (size_t)i * GE::N, nullptr, row, lt,
                                                pick(rp.galois, z), pk);
            else
#pragma unroll
                for (int r = 0; r < 16; ++r) cc[r] = c0v[r];
#pragma unroll
            for (int r = 0; r < 16; ++r) o[r] = red1(o[r] + cc[r], q);
        }
        gstore<PLAST>(o, (h == 0 ? out0 : out1) + z * outz + (size_t)i * GE::N + rowoff, lt);
    };
    half(0);
    half(1);
}

// ------------------------------------------------------------ ModUp finish
// grid (ROW_BLOCKS, l+alpha, beta).  ext[j][t] = c1[t] for t in D_j, else the
// forward row pass (in place) of the column-pass output already in ext[j][t].
template <int LOGN>
__global__ void __launch_bounds__(Geo<LOGN>::ROW_THREADS, ROW_MIN_CTAS)
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

// This file is compiled once per ring degree, with -DPC_LOGN=10..17; its
// launchers live in namespace pc::n<PC_LOGN> (dispatch.cu picks the one of a
// context's ring degree), so every kernel template is instantiated for one
// ring degree per translation unit.
#ifndef PC_LOGN
#error "compile kernels.cu with -DPC_LOGN=<log2 of the ring degree>"
#endif
#define PC_DISPATCH(LOGN_VAR, ...) { constexpr int LG = PC_LOGN; __VA_ARGS__; }
#define PC_NS_CAT2(a, b) a##b
#define PC_NS_CAT(a, b) PC_NS_CAT2(a, b)
#define PC_NS PC_NS_CAT(n, PC_LOGN)

namespace PC_NS {

// shared memory of k_colconv: alpha y tiles and one exchange line per warp
template <class GE>
static size_t colconv_smem(const pc_ctx *c) {
    return sizeof(u32) * ((size_t)c->alpha * GE::CPW * GE::TPCOL * YT_LS + (size_t)c->alpha * GE::CPW * GE::COL_LS4);
}

// k_inner_ws: the key 'b' double buffer, the ring of regenerated 'a'
// buffers, and the counter-free first-round words of each of the beta digits
template <class GE>
static constexpr size_t inner_ws_smem(u32 beta) {
    return row_smem_bytes<GE>(2) + sizeof(u32) * ((2 + WS_RING) * 16 * GE::ROW_THREADS + 12 * (size_t)beta);
}

// k_inner with ROT: the packed source columns, 4 words per thread
template <class GE>
static constexpr size_t inner_rot_extra() {
    return sizeof(u32) * 4 * GE::ROW_THREADS;
}

// the warp-specialised inner product (PC_INNER_WS=0 at the first launch
// selects the single-group kernel, for measurement)
static bool use_inner_ws() {
    static const bool on = [] {
        const char *v = getenv("PC_INNER_WS");
        return !(v && v[0] == '0');
    }();
    return on;
}

template <class F>
static cudaError_t allow_smem(F *f, size_t bytes) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int LG>
static cudaError_t allow_inner_ws() {
    using GE = Geo<LG>;
    if constexpr (LastPhase<GE::LOGC>::type::KK == 16) return allow_smem(k_inner_ws<LG>, inner_ws_smem<GE>(MAX_L));
    else return cudaSuccess;
}

cudaError_t timeline_read(const pc_ctx *c, uint64_t *out) {
    (void)c;
#ifdef PC_TIMELINE
    static_assert(sizeof(g_tl) == sizeof(uint64_t) * PC_TL_ROLES * PC_TL_CTAS * 3, "timeline layout");
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(out, g_tl, sizeof(g_tl));
    void *p = nullptr;
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_tl);
    if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(g_tl));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return e;
#else
    (void)out;
    return cudaErrorNotSupported;
#endif
}

cudaError_t prepare_kernels(pc_ctx *c) {
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        cudaError_t e = allow_smem(k_row<LG, true, false>, row_smem_bytes<GE>(0));
        if (e == cudaSuccess) e = allow_smem(k_row<LG, false, false>, row_smem_bytes<GE>(0));
        if (e == cudaSuccess) e = allow_smem(k_row<LG, false, true>, row_smem_bytes<GE>(1));
        if (e == cudaSuccess) e = allow_smem(k_row<LG, false, true, true>, row_smem_bytes<GE>(1));
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, false, true>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, false, false>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, true, true>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_inner<LG, true, false>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_inner_ws<LG>();
        if (e == cudaSuccess) e = allow_smem(k_inner_rot<LG, true>, row_smem_bytes<GE>(2) + inner_rot_extra<GE>());
        if (e == cudaSuccess) e = allow_smem(k_inner_rot<LG, false>, row_smem_bytes<GE>(2) + inner_rot_extra<GE>());
        if (e == cudaSuccess) e = allow_smem(k_moddown_row<LG, XF_PLAIN>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_moddown_row<LG, XF_GATHER>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_moddown_row<LG, XF_MUL>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_moddown_row<LG, XF_MAC>, row_smem_bytes<GE>(2));
        if (e == cudaSuccess) e = allow_smem(k_modup_finish<LG>, row_smem_bytes<GE>(0));
        if (e == cudaSuccess) e = allow_smem(k_colconv<LG, true>, colconv_smem<GE>(c));
        if (e == cudaSuccess) e = allow_smem(k_colconv<LG, false>, colconv_smem<GE>(c));
        int per_sm = 0, sms = 0;
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_colconv<LG, true>, 32 * c->alpha,
                                                              colconv_smem<GE>(c));
        if (e != cudaSuccess) return e;
        const char *split = getenv("PC_COLCONV_SPLIT");
        c->colconv_slots = split && split[0] == '0' ? 0u : (u32)(per_sm * sms);
    });
    return cudaSuccess;
}

cudaError_t launch_row(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, bool canonical, bool cm_out, cudaStream_t s, u32 galois,
                       const u32 *mul, u32 *xout, const MacIn *mac) {
    if (mac && (fwd || !cm_out || Z != 1 || first_prime != 0)) return cudaErrorInvalidValue;
    const MacIn m = mac ? *mac : MacIn{};
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, nlimbs, Z);
        auto go = [&](auto kern, int tiles) {
            return launch_ex(c, kern, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(tiles), s, c->tab, in, out,
                             first_prime, zin, zout, (int)canonical, galois, mul, xout, m);
        };
        if (fwd) e = go(k_row<LG, true, false>, 0);
        else if (mac) e = go(k_row<LG, false, true, true>, 1);
        else if (cm_out) e = go(k_row<LG, false, true>, 1);
        else e = go(k_row<LG, false, false>, 0);
    });
    return e;
}

cudaError_t launch_col(const pc_ctx *c, bool fwd, const u32 *in, u32 *out, u32 first_prime, u32 nlimbs, u32 Z,
                       size_t zin, size_t zout, int scale_mode, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::COL_BLOCKS, nlimbs, Z);
        if (fwd)
            e = launch_ex(c, k_col<LG, true>, grid, dim3(GE::COL_THREADS), 0, s, c->tab, in, out, first_prime, zin,
                          zout, scale_mode);
        else
            e = launch_ex(c, k_col<LG, false>, grid, dim3(GE::COL_THREADS), 0, s, c->tab, in, out, first_prime, zin,
                          zout, scale_mode);
    });
    return e;
}

// Work split of the conversion kernel.  A CTA's time is mostly the latency of
// its dependent column passes, so a call whose items (unit, strip) fill under
// a quarter of the device's resident CTAs (small rings) splits every item's
// targets over `split` CTAs, each redoing the short source passes: at most 4
// parts, at least alpha targets a part (every warp busy).  Larger calls keep
// whole items (the extra CTAs of a split held the SMs longer than the shorter
// tail saved, and delayed the kernels that overlap the ModUp conversion),
// except the ModDown conversion when its items fill between one and two waves
// (N=2^17: 512 on 444): it runs after the inner products, and the partial
// second wave of whole items would run alone, so it takes halves.
static u32 colconv_split(int mode, u32 items, u32 slots, u32 ntarg, u32 alpha) {
    if (mode == 1 && slots && items > slots && items < 2 * slots && ntarg / 2 >= alpha) return 2;
    if (!slots || 4 * items > slots) return 1;
    u32 k = slots / items;
    if (k > 4) k = 4;
    while (k > 1 && ntarg / k < alpha) --k;
    return k;
}

cudaError_t launch_colconv(const pc_ctx *c, int mode, const u32 *src, size_t srcz, u32 *out, size_t outz, u32 l,
                           u32 Z, bool out_cm, cudaStream_t s) {
    const u32 units = mode == 0 ? (l + c->alpha - 1) / c->alpha : 2;
    // fewest targets of a unit: l + alpha - d with d <= min(alpha, l) (ModUp), or l (ModDown)
    const u32 ntarg = mode == 0 ? (l > c->alpha ? l : c->alpha) : l;
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        const u32 items = (u32)(GE::C / GE::CPW) * units * Z;
        const u32 split = colconv_split(mode, items, c->colconv_slots, ntarg, c->alpha);
        const dim3 grid(items * split);
        if (out_cm)
            e = launch_ex(c, k_colconv<LG, true>, grid, dim3(32 * c->alpha), colconv_smem<GE>(c), s, c->tab, mode,
                          src, srcz, out, outz, l, split);
        else
            e = launch_ex(c, k_colconv<LG, false>, grid, dim3(32 * c->alpha), colconv_smem<GE>(c), s, c->tab, mode,
                          src, srcz, out, outz, l, split);
    });
    return e;
}

// the two-group inner product where a thread's 16 coefficients are two whole
// ChaCha blocks (rows of 256 words, N >= 2^12); instantiated only there
template <int LG>
static cudaError_t launch_inner_ws(const pc_ctx *c, dim3 grid, cudaStream_t s, const u32 *src, size_t srcz,
                                   const u32 *c1, size_t c1z, u32 *acc, size_t accz, u32 l, const KeyPack &kp,
                                   int pi, u32 t0) {
    using GE = Geo<LG>;
    if constexpr (LastPhase<GE::LOGC>::type::KK == 16)
        return launch_ex(c, k_inner_ws<LG>, grid, dim3(2 * GE::ROW_THREADS),
                         inner_ws_smem<GE>((l + c->alpha - 1) / c->alpha), s, c->tab, src, srcz, c1, c1z, acc, accz,
                         l, kp, pi, t0);
    else
        return cudaErrorInvalidValue;
}

cudaError_t launch_inner(const pc_ctx *c, bool fused, const u32 *src, size_t srcz, const u32 *c1, size_t c1z,
                         u32 *acc, size_t accz, u32 l, const KeyPack &kp, u32 Z, bool regen, bool pintt,
                         cudaStream_t s, u32 t0, u32 nt, const RotPack *rot) {
    if (rot && (!fused || Z > (u32)KEYS_PER_LAUNCH)) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (nt == 0) nt = l + c->alpha - t0;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, nt, Z);
        const size_t sm = row_smem_bytes<GE>(2) + (rot ? inner_rot_extra<GE>() : 0);
        const int pi = pintt ? 1 : 0;
        // the two-group kernel needs a thread's 16 coefficients to be two
        // whole ChaCha blocks (rows of 256 words: N >= 2^12)
        constexpr bool ws_ok = LastPhase<GE::LOGC>::type::KK == 16;
        auto go = [&](auto kern) {
            return launch_ex(c, kern, grid, dim3(GE::ROW_THREADS), sm, s, c->tab, src, srcz, c1, c1z, acc, accz, l,
                             kp, pi, t0);
        };
        auto go_rot = [&](auto kern) {
            return launch_ex(c, kern, grid, dim3(GE::ROW_THREADS), sm, s, c->tab, src, srcz, c1, c1z, acc, accz, l,
                             kp, pi, t0, *rot);
        };
        if (rot) e = regen ? go_rot(k_inner_rot<LG, true>) : go_rot(k_inner_rot<LG, false>);
        else if (fused && regen && use_inner_ws() && ws_ok)
            e = launch_inner_ws<LG>(c, grid, s, src, srcz, c1, c1z, acc, accz, l, kp, pi, t0);
        else if (fused) e = regen ? go(k_inner<LG, true, true>) : go(k_inner<LG, true, false>);
        else e = regen ? go(k_inner<LG, false, true>) : go(k_inner<LG, false, false>);
    });
    return e;
}

cudaError_t launch_moddown_row(const pc_ctx *c, const u32 *U, size_t Uz, const u32 *acc, size_t accz, const u32 *c0,
                               size_t c0z, u32 *out0, u32 *out1, size_t outz, u32 l, u32 Z, cudaStream_t s,
                               const RotPack *rot, const u32 *rx, const u32 *ry, const MacIn *mac) {
    if (rot && Z > (u32)KEYS_PER_LAUNCH) return cudaErrorInvalidValue;
    if (mac && (Z != 1 || rx)) return cudaErrorInvalidValue;
    const MacIn m = mac ? *mac : MacIn{};
    RotPack rp{};
    for (int z = 0; z < KEYS_PER_LAUNCH; ++z) rp.galois[z] = rp.ginv[z] = 1;
    if (rot) rp = *rot;
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l, Z);
        auto go = [&](auto kern) {
            return launch_ex(c, kern, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(2), s, c->tab, U, Uz, acc,
                             accz, c0, c0z, out0, out1, outz, l, rp, rx, ry, m);
        };
        if (mac) e = go(k_moddown_row<LG, XF_MAC>);
        else if (rx) e = Z == 1 && ry ? go(k_moddown_row<LG, XF_MUL>) : cudaErrorInvalidValue;
        else if (rot) e = go(k_moddown_row<LG, XF_GATHER>);
        else e = go(k_moddown_row<LG, XF_PLAIN>);
    });
    return e;
}

cudaError_t launch_modup_finish(const pc_ctx *c, const u32 *c1, u32 *ext, u32 l, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    PC_DISPATCH(c->logN, {
        using GE = Geo<LG>;
        dim3 grid(GE::ROW_BLOCKS, l + c->alpha, (l + c->alpha - 1) / c->alpha);
        e = launch_ex(c, k_modup_finish<LG>, grid, dim3(GE::ROW_THREADS), row_smem_bytes<GE>(0), s, c->tab, c1, ext,
                      l);
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

}  // namespace n<PC_LOGN>
}  // namespace pc
