// ntt.cuh -- negacyclic NTT building blocks for sm_100a.
//
// Transform (spec v1; Longa-Naehrig merged-psi Cooley-Tukey network):
//   a_hat[k] = sum_n a[n] psi^((2 brv(k) + 1) n) mod q, bit-reversed order.
// Stage s (0-based) pairs elements at distance N >> (s+1); the butterfly whose
// lower element is X uses psi_rev[(1 << s) + (X >> (logN - s))], with
// psi_rev[k] = psi^brv(k).  The inverse runs the stages backwards with
// Gentleman-Sande butterflies and psi^-1 powers, then scales by N^-1.
//
// B200 decomposition: N = R x C viewed as R rows of C contiguous words.
//   - stages 0..logR-1 only pair elements of the same column: the "column
//     pass", R-point transforms on C columns, every column using the same
//     twiddles psi_rev[1..R-1];
//   - stages logR..logN-1 stay inside a row: the "row pass", C-point
//     transforms whose row-r twiddle for local stage s and group i is
//     psi_rev[(R + r) 2^s + i]; they are re-laid out per row as
//     RT[r][(1 << s) + i] so one row's table is C contiguous entries.
// Every pass is a "line transform" of length M = 2^m (M = R or C): each
// thread keeps 16 elements in registers and runs up to four stages (one
// radix-16 phase) on them; phases exchange through shared memory.  A line
// of M elements is handled by M/16 threads.
#pragma once
#include <type_traits>

#include "modarith.cuh"

namespace pc {

// One phase: stages [S0, S0+K) of a length-2^LOGM line transform.
// Register r = g*2^K + m holds element x_of(lt, r) of the thread's line.
template <int LOGM, int S0, int K>
struct Phase {
    static constexpr int M = 1 << LOGM;
    static constexpr int LOGD = LOGM - S0 - K;  // smallest distance of the phase
    static constexpr int D = 1 << LOGD;
    static constexpr int KK = 1 << K;  // members per group
    static constexpr int G = 16 / KK;  // groups per thread
    static constexpr int T = M / 16;   // threads per line
    static_assert(K >= 1 && K <= 4 && LOGD >= 0, "bad phase");

    __device__ static __forceinline__ int pair(int lt, int g) { return lt + g * T; }
    __device__ static __forceinline__ int x_of(int lt, int r) {
        const int g = r / KK, m = r % KK;
        const int p = pair(lt, g);
        return ((p >> LOGD) << (LOGD + K)) + (m << LOGD) + (p & (D - 1));
    }

    // forward stages; tw(s, u, hi, b) returns {w, w'} for the table entry
    // (1 << s) + (hi << u) + b of stage s = S0 + u (natural layout; see TwRow for the stored one)
    template <class TW>
    __device__ static __forceinline__ void fwd(u32 v[16], int lt, const TW &tw, u32 q) {
#pragma unroll
        for (int u = 0; u < K; ++u) {
            const int h = KK >> (u + 1);  // member distance at this sub-stage
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int hi = pair(lt, g) >> LOGD;
#pragma unroll
                for (int b = 0; b < (1 << u); ++b) {
                    const uint2 w = tw(S0 + u, u, hi, b);
#pragma unroll
                    for (int a = b * (KK >> u); a < b * (KK >> u) + h; ++a)
                        bf_ct(v[g * KK + a], v[g * KK + a + h], w.x, w.y, q);
                }
            }
        }
    }

    template <class TW>
    __device__ static __forceinline__ void inv(u32 v[16], int lt, const TW &tw, u32 q) {
#pragma unroll
        for (int u = K - 1; u >= 0; --u) {
            const int h = KK >> (u + 1);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int hi = pair(lt, g) >> LOGD;
#pragma unroll
                for (int b = 0; b < (1 << u); ++b) {
                    const uint2 w = tw(S0 + u, u, hi, b);
#pragma unroll
                    for (int a = b * (KK >> u); a < b * (KK >> u) + h; ++a)
                        bf_gs(v[g * KK + a], v[g * KK + a + h], w.x, w.y, q);
                }
            }
        }
    }
};

// Phase partition of a length-2^LOGM line: [0,4), [4,8), [8,LOGM).
template <int LOGM>
struct Plan {
    static_assert(LOGM >= 4 && LOGM <= 9, "line length 16..512");
    static constexpr int NPH = LOGM <= 4 ? 1 : (LOGM <= 8 ? 2 : 3);
    using P0 = Phase<LOGM, 0, (LOGM < 4 ? LOGM : 4)>;
    using P1 = Phase<LOGM, 4, (LOGM > 4 ? (LOGM - 4 < 4 ? LOGM - 4 : 4) : 1)>;
    using P2 = Phase<LOGM, 8, (LOGM > 8 ? LOGM - 8 : 1)>;
    // element held by register r at the start / end of a forward transform
    __device__ static __forceinline__ int fwd_in(int lt, int r) { return P0::x_of(lt, r); }
    __device__ static __forceinline__ int fwd_out(int lt, int r) {
        if constexpr (NPH == 1) return P0::x_of(lt, r);
        else if constexpr (NPH == 2) return P1::x_of(lt, r);
        else return P2::x_of(lt, r);
    }
    // the inverse starts where the forward ends and ends where it starts
    __device__ static __forceinline__ int inv_in(int lt, int r) { return fwd_out(lt, r); }
    __device__ static __forceinline__ int inv_out(int lt, int r) { return fwd_in(lt, r); }
};

// Barriers that order a line's shared-memory exchange: a warp barrier when
// every line's threads sit in one warp, else a CTA barrier.
struct SyncWarp {
    __device__ __forceinline__ void operator()() const { __syncwarp(); }
};
struct SyncCta {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// Line layout with 16-byte exchanges: element x at x + 4 (x >> 4).  A lane's
// run of 16 consecutive elements (a distance-1 phase) is then four aligned
// 16-byte chunks, and with runs 20 words apart any 8 consecutive lanes' chunks
// fall on distinct bank groups; a strided phase (elements lt + 16 r) touches
// one word per lane, consecutive lanes on consecutive banks.  Lines need
// M + M/4 words.
struct Pad4Addr {
    __device__ __forceinline__ int operator()(int x) const { return x + 4 * (x >> 4); }
};

template <class PH>
struct IsRun16 {  // a thread holds 16 consecutive elements of the line
    static constexpr bool value = PH::D == 1 && PH::KK == 16;
};

// Exchange the registers of phase A's layout into phase B's layout through
// shared memory.  ADDR(x) gives the word address of element x of the line.
template <class PA, class PB, class SYNC, class ADDR>
__device__ __forceinline__ void exchange(u32 v[16], u32 *sm, int lt, const ADDR &addr, const SYNC &sync) {
    constexpr bool pad4 = std::is_same<ADDR, Pad4Addr>::value;
    sync();
    if constexpr (pad4 && IsRun16<PA>::value) {
        uint4 *d = reinterpret_cast<uint4 *>(sm + addr(PA::x_of(lt, 0)));
#pragma unroll
        for (int c = 0; c < 4; ++c) d[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) sm[addr(PA::x_of(lt, r))] = v[r];
    }
    sync();
    if constexpr (pad4 && IsRun16<PB>::value) {
        const uint4 *d = reinterpret_cast<const uint4 *>(sm + addr(PB::x_of(lt, 0)));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w = d[c];
            v[4 * c] = w.x; v[4 * c + 1] = w.y; v[4 * c + 2] = w.z; v[4 * c + 3] = w.w;
        }
    } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = sm[addr(PB::x_of(lt, r))];
    }
}

// Full forward line transform: registers enter at Plan::fwd_in positions and
// leave at Plan::fwd_out positions (lazy values in [0, 2q)).
template <int LOGM, class ADDR, class TW, class SYNC>
__device__ __forceinline__ void line_fwd(u32 v[16], u32 *sm, int lt, const ADDR &addr, const TW &tw, u32 q,
                                         const SYNC &sync) {
    using PL = Plan<LOGM>;
    PL::P0::fwd(v, lt, tw, q);
    if constexpr (PL::NPH >= 2) {
        exchange<typename PL::P0, typename PL::P1>(v, sm, lt, addr, sync);
        PL::P1::fwd(v, lt, tw, q);
    }
    if constexpr (PL::NPH >= 3) {
        exchange<typename PL::P1, typename PL::P2>(v, sm, lt, addr, sync);
        PL::P2::fwd(v, lt, tw, q);
    }
}

// Full inverse line transform (no N^-1): registers enter at Plan::inv_in
// and leave at Plan::inv_out positions.
template <int LOGM, class ADDR, class TW, class SYNC>
__device__ __forceinline__ void line_inv(u32 v[16], u32 *sm, int lt, const ADDR &addr, const TW &tw, u32 q,
                                         const SYNC &sync) {
    using PL = Plan<LOGM>;
    if constexpr (PL::NPH >= 3) {
        PL::P2::inv(v, lt, tw, q);
        exchange<typename PL::P2, typename PL::P1>(v, sm, lt, addr, sync);
    }
    if constexpr (PL::NPH >= 2) {
        PL::P1::inv(v, lt, tw, q);
        exchange<typename PL::P1, typename PL::P0>(v, sm, lt, addr, sync);
    }
    PL::P0::inv(v, lt, tw, q);
}

// Twiddle tables as stored on the device ("re-laid"): within stage s, with
// u = s mod 4 and S0 = s - u (the first stage of its radix-16 phase), the
// natural entry (1 << s) + (hi << u) + b sits at (1 << s) + (b << S0) + hi.
// At fixed b the threads of one line (consecutive hi) then read consecutive
// entries: coalesced from global memory, free of shared-memory bank
// conflicts.  Stages 0..3 keep the natural order (hi = 0 there: the whole
// line shares those twiddles).
struct TwRow {
    const uint2 *t;
    __device__ __forceinline__ uint2 operator()(int s, int u, int hi, int b) const {
        return t[(1 << s) + (b << (s - u)) + hi];
    }
};
// The same tables read through the read-only data path.
struct TwRowG {
    const uint2 *t;
    __device__ __forceinline__ uint2 operator()(int s, int u, int hi, int b) const {
        return __ldg(t + (1 << s) + (b << (s - u)) + hi);
    }
};

// 16-byte asynchronous global -> shared copy (bypasses registers and L1)
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Named hardware barriers (ids 1..15; id 0 is __syncthreads): bar_sync
// waits until `count` threads (a multiple of 32) have arrived at barrier id
// in this phase, bar_arrive arrives without waiting.  Shared-memory writes made
// before an arrive are visible to the threads that pass the matching sync.
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

// Programmatic dependent launch: pdl_wait() blocks until the previous grid on
// the stream has completed and its writes are visible (a no-op when the
// kernel was launched without the attribute); pdl_trigger() lets the next
// grid start launching once every CTA of this grid has called it.  Kernels
// read only constant tables (and the ModDown finish the caller's c0, which no
// kernel of a call writes) before pdl_wait() and write nothing before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" :::); }

// Geometry of a ring of degree 2^LOGN_: C = 2^LOGC-word rows, R = 2^LOGR rows.
template <int LOGN_>
struct Geo {
    static constexpr int LOGN = LOGN_;
    static constexpr int LOGC = (LOGN - 4 < 8) ? LOGN - 4 : 8;
    static constexpr int LOGR = LOGN - LOGC;
    static constexpr int N = 1 << LOGN, C = 1 << LOGC, R = 1 << LOGR;
    // row pass: NL = 8 rows per CTA (a 32-byte segment of every column of a
    // column-major limb), C/16 threads per row
    static constexpr int TPR = C / 16;
    static constexpr int NL = 8;
    static constexpr int ROW_THREADS = NL * TPR;
    static constexpr int ROW_BLOCKS = R / NL;
    static constexpr int ROW_LS = C + C / 16;  // padded row stride in shared memory
    // column pass on a row-major limb (the NTT calls): W columns per CTA,
    // R/16 threads per column, CTA barriers between phases; the shared tile
    // is row-major with one W-word pad every 16 rows
    static constexpr int TPCOL = R / 16;
    static constexpr int W_ = 2048 / R > 4 ? 2048 / R : 4;
    static constexpr int W = W_ < C ? W_ : C;
    static constexpr int COL_THREADS = W * TPCOL;
    static constexpr int COL_BLOCKS = C / W;
    static constexpr int COL_TILE = (R + R / 16) * W;  // words of the padded tile
    // column pass on a column-major limb (the key-switch kernels): one column
    // per TPCOL consecutive lanes, CPW columns per warp, warp barriers only
    static constexpr int CPW = 32 / TPCOL;
    static constexpr int COL_LS = R + R / 16;  // padded column stride in shared memory
    // column stride of a Pad4Addr line (+16 words: a warp's two columns on
    // opposite bank halves)
    static constexpr int COL_LS4 = R + R / 4 + 16;
    static_assert(LOGC >= 4 && LOGR >= 4 && LOGR <= 9, "supported 2^8..2^17 (R,C >= 16)");
};

}  // namespace pc
