// chacha.cuh -- ChaCha12 block function in registers (Bernstein 2008).
//
// Used to regenerate the uniform 'a' half of a key-switching key inside the
// inner-product kernel instead of reading it from HBM (Perseus README, "What's
// inside": in-kernel key regeneration from a ChaCha12 seed; arxivlens summary
// of the Perseus paper, "Methodology": ChaCha12 counter-mode expander).
//
// Spec v1 state: words 0..3 "expand 32-byte k", 4..11 the 32-byte seed as
// little-endian words, 12 the block counter, 13 the global prime index,
// 14 the digit, 15 the tag 0x61.  Six double rounds, then the input state is
// added word-wise.
#pragma once
#include <cstdint>

namespace pc {

__device__ __forceinline__ uint32_t rotl32(uint32_t x, int r) { return __funnelshift_l(x, x, r); }

// Rotation on the integer multiply pipe: for m = 2^r (kept opaque to the
// compiler), x*m + umulhi(x, m) = (x << r) | (x >> (32 - r)).  Used for some
// rotations to balance the ALU pipe (xor, funnel shift) against the
// multiply-add pipe.
__device__ __forceinline__ uint32_t rotl_mul(uint32_t x, uint32_t m) { return x * m + __umulhi(x, m); }

// Which of the four quarter-round rotations (16, 12, 8, 7) run on the
// multiply pipe: bit i set -> rotation i uses rotl_mul with mul[i] = 2^r.
template <int MULMASK>
struct ChaRot {
    uint32_t mul[4];
    __device__ __forceinline__ uint32_t r(int i, uint32_t x) const {
        const int amt[4] = {16, 12, 8, 7};
        return ((MULMASK >> i) & 1) ? rotl_mul(x, mul[i]) : rotl32(x, amt[i]);
    }
};

// Byte-aligned rotations (16 and 8) as byte permutes, the others as funnel
// shifts.
struct ChaRotPrmt {
    __device__ __forceinline__ uint32_t r(int i, uint32_t x) const {
        if (i == 0) return __byte_perm(x, x, 0x1032);
        if (i == 2) return __byte_perm(x, x, 0x2103);
        return rotl32(x, i == 1 ? 12 : 7);
    }
};

#define PC_QR(a, b, c, d)                          \
    a += b; d ^= a; d = R.r(0, d);                 \
    c += d; b ^= c; b = R.r(1, b);                 \
    a += b; d ^= a; d = R.r(2, d);                 \
    c += d; b ^= c; b = R.r(3, b);

// out[16] = ChaCha12(seed words k[8], counter, g, j)
template <class ROT = ChaRot<0>>
__device__ __forceinline__ void chacha12_block(const uint32_t k[8], uint32_t ctr, uint32_t g, uint32_t j,
                                               uint32_t out[16], const ROT &R = ROT{}) {
    const uint32_t c0 = 0x61707865u, c1 = 0x3320646eu, c2 = 0x79622d32u, c3 = 0x6b206574u;
    uint32_t x0 = c0, x1 = c1, x2 = c2, x3 = c3;
    uint32_t x4 = k[0], x5 = k[1], x6 = k[2], x7 = k[3];
    uint32_t x8 = k[4], x9 = k[5], x10 = k[6], x11 = k[7];
    uint32_t x12 = ctr, x13 = g, x14 = j, x15 = 0x61u;
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        PC_QR(x0, x4, x8, x12);
        PC_QR(x1, x5, x9, x13);
        PC_QR(x2, x6, x10, x14);
        PC_QR(x3, x7, x11, x15);
        PC_QR(x0, x5, x10, x15);
        PC_QR(x1, x6, x11, x12);
        PC_QR(x2, x7, x8, x13);
        PC_QR(x3, x4, x9, x14);
    }
    out[0] = x0 + c0; out[1] = x1 + c1; out[2] = x2 + c2; out[3] = x3 + c3;
    out[4] = x4 + k[0]; out[5] = x5 + k[1]; out[6] = x6 + k[2]; out[7] = x7 + k[3];
    out[8] = x8 + k[4]; out[9] = x9 + k[5]; out[10] = x10 + k[6]; out[11] = x11 + k[7];
    out[12] = x12 + ctr; out[13] = x13 + g; out[14] = x14 + j; out[15] = x15 + 0x61u;
}
// Two blocks (counters ctr and ctr + 1) with their quarter rounds
// interleaved: twice the independent dependency chains per thread.
__device__ __forceinline__ void chacha12_block2(const uint32_t k[8], uint32_t ctr, uint32_t g, uint32_t j,
                                                uint32_t o0[16], uint32_t o1[16]) {
    const uint32_t c0 = 0x61707865u, c1 = 0x3320646eu, c2 = 0x79622d32u, c3 = 0x6b206574u;
    const ChaRot<0> R{};
    uint32_t x0 = c0, x1 = c1, x2 = c2, x3 = c3, x4 = k[0], x5 = k[1], x6 = k[2], x7 = k[3];
    uint32_t x8 = k[4], x9 = k[5], x10 = k[6], x11 = k[7], x12 = ctr, x13 = g, x14 = j, x15 = 0x61u;
    uint32_t y0 = c0, y1 = c1, y2 = c2, y3 = c3, y4 = k[0], y5 = k[1], y6 = k[2], y7 = k[3];
    uint32_t y8 = k[4], y9 = k[5], y10 = k[6], y11 = k[7], y12 = ctr + 1, y13 = g, y14 = j, y15 = 0x61u;
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        PC_QR(x0, x4, x8, x12);
        PC_QR(y0, y4, y8, y12);
        PC_QR(x1, x5, x9, x13);
        PC_QR(y1, y5, y9, y13);
        PC_QR(x2, x6, x10, x14);
        PC_QR(y2, y6, y10, y14);
        PC_QR(x3, x7, x11, x15);
        PC_QR(y3, y7, y11, y15);
        PC_QR(x0, x5, x10, x15);
        PC_QR(y0, y5, y10, y15);
        PC_QR(x1, x6, x11, x12);
        PC_QR(y1, y6, y11, y12);
        PC_QR(x2, x7, x8, x13);
        PC_QR(y2, y7, y8, y13);
        PC_QR(x3, x4, x9, x14);
        PC_QR(y3, y4, y9, y14);
    }
    o0[0] = x0 + c0; o0[1] = x1 + c1; o0[2] = x2 + c2; o0[3] = x3 + c3;
    o0[4] = x4 + k[0]; o0[5] = x5 + k[1]; o0[6] = x6 + k[2]; o0[7] = x7 + k[3];
    o0[8] = x8 + k[4]; o0[9] = x9 + k[5]; o0[10] = x10 + k[6]; o0[11] = x11 + k[7];
    o0[12] = x12 + ctr; o0[13] = x13 + g; o0[14] = x14 + j; o0[15] = x15 + 0x61u;
    o1[0] = y0 + c0; o1[1] = y1 + c1; o1[2] = y2 + c2; o1[3] = y3 + c3;
    o1[4] = y4 + k[0]; o1[5] = y5 + k[1]; o1[6] = y6 + k[2]; o1[7] = y7 + k[3];
    o1[8] = y8 + k[4]; o1[9] = y9 + k[5]; o1[10] = y10 + k[6]; o1[11] = y11 + k[7];
    o1[12] = y12 + ctr + 1; o1[13] = y13 + g; o1[14] = y14 + j; o1[15] = y15 + 0x61u;
}
// The first column round's quarter rounds on columns 1, 2 and 3 do not touch
// the block counter (word 12): for a fixed seed, prime index and digit they
// are the same in every block.  pre[12] = words 1, 5, 9, 13, 2, 6, 10, 14,
// 3, 7, 11, 15 after them.
__device__ __forceinline__ void chacha12_precolumn(const uint32_t k[8], uint32_t g, uint32_t j, uint32_t pre[12]) {
    const ChaRot<0> R{};
    uint32_t x1 = 0x3320646eu, x5 = k[1], x9 = k[5], x13 = g;
    uint32_t x2 = 0x79622d32u, x6 = k[2], x10 = k[6], x14 = j;
    uint32_t x3 = 0x6b206574u, x7 = k[3], x11 = k[7], x15 = 0x61u;
    PC_QR(x1, x5, x9, x13);
    PC_QR(x2, x6, x10, x14);
    PC_QR(x3, x7, x11, x15);
    pre[0] = x1; pre[1] = x5; pre[2] = x9; pre[3] = x13;
    pre[4] = x2; pre[5] = x6; pre[6] = x10; pre[7] = x14;
    pre[8] = x3; pre[9] = x7; pre[10] = x11; pre[11] = x15;
}

// Blocks ctr and ctr + 1 (interleaved) starting from chacha12_precolumn's
// words: the remaining quarter round of the first column round, then the
// rest of the six double rounds, then the feed-forward of the input state.
__device__ __forceinline__ void chacha12_block2_pre(const uint32_t pre[12], const uint32_t k[8], uint32_t ctr,
                                                    uint32_t g, uint32_t j, uint32_t o0[16], uint32_t o1[16]) {
    const uint32_t c0 = 0x61707865u, c1 = 0x3320646eu, c2 = 0x79622d32u, c3 = 0x6b206574u;
    const ChaRot<0> R{};
    uint32_t x0 = c0, x4 = k[0], x8 = k[4], x12 = ctr;
    uint32_t y0 = c0, y4 = k[0], y8 = k[4], y12 = ctr + 1;
    uint32_t x1 = pre[0], x5 = pre[1], x9 = pre[2], x13 = pre[3];
    uint32_t x2 = pre[4], x6 = pre[5], x10 = pre[6], x14 = pre[7];
    uint32_t x3 = pre[8], x7 = pre[9], x11 = pre[10], x15 = pre[11];
    uint32_t y1 = x1, y5 = x5, y9 = x9, y13 = x13, y2 = x2, y6 = x6, y10 = x10, y14 = x14;
    uint32_t y3 = x3, y7 = x7, y11 = x11, y15 = x15;
    PC_QR(x0, x4, x8, x12);
    PC_QR(y0, y4, y8, y12);
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        if (i > 0) {
            PC_QR(x0, x4, x8, x12);
            PC_QR(y0, y4, y8, y12);
            PC_QR(x1, x5, x9, x13);
            PC_QR(y1, y5, y9, y13);
            PC_QR(x2, x6, x10, x14);
            PC_QR(y2, y6, y10, y14);
            PC_QR(x3, x7, x11, x15);
            PC_QR(y3, y7, y11, y15);
        }
        PC_QR(x0, x5, x10, x15);
        PC_QR(y0, y5, y10, y15);
        PC_QR(x1, x6, x11, x12);
        PC_QR(y1, y6, y11, y12);
        PC_QR(x2, x7, x8, x13);
        PC_QR(y2, y7, y8, y13);
        PC_QR(x3, x4, x9, x14);
        PC_QR(y3, y4, y9, y14);
    }
    o0[0] = x0 + c0; o0[1] = x1 + c1; o0[2] = x2 + c2; o0[3] = x3 + c3;
    o0[4] = x4 + k[0]; o0[5] = x5 + k[1]; o0[6] = x6 + k[2]; o0[7] = x7 + k[3];
    o0[8] = x8 + k[4]; o0[9] = x9 + k[5]; o0[10] = x10 + k[6]; o0[11] = x11 + k[7];
    o0[12] = x12 + ctr; o0[13] = x13 + g; o0[14] = x14 + j; o0[15] = x15 + 0x61u;
    o1[0] = y0 + c0; o1[1] = y1 + c1; o1[2] = y2 + c2; o1[3] = y3 + c3;
    o1[4] = y4 + k[0]; o1[5] = y5 + k[1]; o1[6] = y6 + k[2]; o1[7] = y7 + k[3];
    o1[8] = y8 + k[4]; o1[9] = y9 + k[5]; o1[10] = y10 + k[6]; o1[11] = y11 + k[7];
    o1[12] = y12 + ctr + 1; o1[13] = y13 + g; o1[14] = y14 + j; o1[15] = y15 + 0x61u;
}
#undef PC_QR

}  // namespace pc
