// modarith.cuh -- 32-bit modular arithmetic for primes q < 2^31 on sm_100a.
//
// Representations: "canonical" = [0, q); "lazy" = [0, 2q) (fits in 32 bits
// because q < 2^31).  Multiplication by a constant w uses Shoup's method with
// the precomputed companion w' = floor(w 2^32 / q) (Shoup; Harvey 2014,
// "Faster arithmetic for number-theoretic transforms"); 64-bit sums are
// reduced with Montgomery's REDC (Montgomery 1985) with R = 2^32.
#pragma once
#include <cstdint>

namespace pc {

typedef uint32_t u32;
typedef uint64_t u64;

// [0, 2q) -> [0, q): x - q wraps to a large value when x < q.
__device__ __forceinline__ u32 red1(u32 x, u32 q) { return min(x, x - q); }

// Shoup: x * w mod q for any x < 2^32, result in [0, 2q).
__device__ __forceinline__ u32 shoup_lazy(u32 x, u32 w, u32 ws, u32 q) {
    u32 qh = __umulhi(x, ws);
    return x * w - qh * q;
}
__device__ __forceinline__ u32 shoup(u32 x, u32 w, u32 ws, u32 q) {
    return red1(shoup_lazy(x, w, ws, q), q);
}

// x mod q for any 32-bit x (Shoup with w = 1, companion floor(2^32/q)).
__device__ __forceinline__ u32 mod32(u32 x, u32 q, u32 q1s) {
    return red1(x - __umulhi(x, q1s) * q, q);
}

// REDC: for x = hi*2^32 + lo with hi < q, returns x * 2^-32 mod q in [0, q).
// qn = -q^-1 mod 2^32.  (x + m q) / 2^32 = hi + umulhi(m, q) + carry, and the
// low-word sum lo + lo(m q) is 0 mod 2^32, so the carry is (lo != 0).
__device__ __forceinline__ u32 redc(u32 lo, u32 hi, u32 q, u32 qn) {
    u32 m = lo * qn;
    u32 r;
    asm("{\n\t.reg .u32 t;\n\t"
        "mad.lo.cc.u32 t, %1, %2, %3;\n\t"
        "madc.hi.u32 %0, %1, %2, %4;\n\t}"
        : "=r"(r)
        : "r"(m), "r"(q), "r"(lo), "r"(hi));
    return red1(r, q);
}

// Exact (x mod q) * 2^-32 for any 64-bit x: fold the high word below q first.
__device__ __forceinline__ u32 redc64(u64 x, u32 q, u32 qn, u32 q1s) {
    u32 hi = mod32((u32)(x >> 32), q, q1s);
    return redc((u32)x, hi, q, qn);
}

// 64-bit accumulator fold: keeps the value mod q unchanged and makes the high
// word < q, so that up to three more products below 2^62 can be added.
__device__ __forceinline__ u64 fold64(u64 x, u32 q, u32 q1s) {
    u32 hi = mod32((u32)(x >> 32), q, q1s);
    return ((u64)hi << 32) | (u32)x;
}

// Forward (Cooley-Tukey) butterfly on lazy inputs; outputs lazy.
//   (a, b) -> (a + w b, a - w b)
__device__ __forceinline__ void bf_ct(u32 &a, u32 &b, u32 w, u32 ws, u32 q) {
    u32 u = red1(a, q);
    u32 t = shoup(b, w, ws, q);
    a = u + t;
    b = u - t + q;
}

// Inverse (Gentleman-Sande) butterfly on lazy inputs; outputs lazy.
//   (a, b) -> (a + b, (a - b) w)
__device__ __forceinline__ void bf_gs(u32 &a, u32 &b, u32 w, u32 ws, u32 q) {
    u32 u = red1(a, q);
    u32 v = red1(b, q);
    a = u + v;
    b = shoup_lazy(u - v + q, w, ws, q);
}

}  // namespace pc
