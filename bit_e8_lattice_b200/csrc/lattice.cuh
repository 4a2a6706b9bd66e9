// Device-side E8 arithmetic: nearest point, core rank, escape root, exact
// bf16 dequantisation.  All lattice points are in doubled coordinates
// P = 2p (integers; all even or all odd; sum divisible by 4).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace e8q {

// Nearest E8 point of x, given X = 2x (fp32), following Conway & Sloane's
// decoder for E8 = D8 u (D8 + 1/2) ("E8-QAT", abstract and Figure 2 (b):
// arithmetic projection with no stored codebook).
//
// One rounding of X to the nearest even integer E gives both cosets at
// once: the D8 coordinate is E/2 (error t = |X - E| <= 1, doubled units)
// and the D8+1/2 coordinate is the odd integer E +- 1 on X's side (error
// 1 - t).  The parity fixes move the coordinate with the largest error
// (lowest index on ties) two steps towards X, which adds 4 - 4*t_max (D8)
// or 4*t_min (D8+1/2) to the squared distance, so both candidate
// distances are known before either point is built.  A distance tie
// keeps the D8 point.  |X| must be below 2^21.
__device__ __forceinline__ void e8_nearest_doubled(const float (&X)[8], int (&P)[8]) {
    const float kMagic = 25165824.0f;  // 1.5 * 2^24: spacing 2, so X + kMagic rounds to an even integer
    const unsigned kMagicBits = 0x4BC00000u;
    int E[8];
    bool neg[8];
    float da = 0.f, st = 0.f, tmax = -1.f, tmin = 4.f;
    int imax = 0, imin = 0, sumh = 0, nneg = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float g = X[i] + kMagic;
        int eh = static_cast<int>(__float_as_uint(g) - kMagicBits);  // E/2, exact
        float e = X[i] - (g - kMagic);                                // X - E in [-1, 1]
        E[i] = 2 * eh;
        sumh += eh;
        neg[i] = e < 0.f;
        nneg += neg[i] ? 1 : 0;
        float t = fabsf(e);
        da = fmaf(e, e, da);
        st += t;
        if (t > tmax) { tmax = t; imax = i; }
        if (t < tmin) { tmin = t; imin = i; }
    }
    const bool oddA = (sumh & 1) != 0;           // sum(E)/2 odd: sum(E) = 2 mod 4
    const bool oddB = ((sumh ^ nneg) & 1) != 0;  // sum(E +- 1) = 2 mod 4
    const float DA = da + (oddA ? (4.f - 4.f * tmax) : 0.f);
    const float DB = (8.f - 2.f * st + da) + (oddB ? 4.f * tmin : 0.f);
    const bool useB = DB < DA;
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = useB ? (E[i] + (neg[i] ? -1 : 1)) : E[i];
    if (useB ? oddB : oddA) {
        const int k = useB ? imin : imax;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i == k) P[i] += (X[i] >= static_cast<float>(P[i])) ? 2 : -2;
    }
}

// Core index of P, or -1 when P is not in the core (tables.h explains the
// two-table decomposition).  t1/t2 may live in shared or global memory.
__device__ __forceinline__ int core_rank(const int (&P)[8], const uint16_t* __restrict__ t1,
                                         const uint16_t* __restrict__ t2) {
    int n2 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) n2 += P[i] * P[i];
    if (n2 > 48) return -1;
    const int type = P[0] & 1;
    int hk = 0, lk = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        hk = hk * 7 + ((P[i] + 6) >> 1);
        lk = lk * 7 + ((P[i + 4] + 6) >> 1);
    }
    const int a = t1[(type * 2401 + hk) * 7 + (n2 >> 3)];
    const int b = t2[type * 2401 + lk];
    const int r = a + b;
    return (a != 0xFFFF && r < 65536) ? r : -1;
}

// The root R (doubled: +-2 at two places, or +-1 everywhere with an even
// number of minus signs) whose core point P - R comes first in the core
// order: largest <P, R> (smallest |P - R|^2), then lexicographically
// largest R (lexicographically smallest P - R).  If that point is outside
// the core, no root puts P into the core, since every other candidate
// comes later in the order.  This picks the escape record of "E8-QAT"
// Figure 2 (c) / Table 3 (core point plus one root).
__device__ __forceinline__ void best_escape_root(const int (&P)[8], int (&R)[8]) {
    int w[8], s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w[i] = abs(P[i]);
        s[i] = P[i] < 0 ? -1 : 1;  // a zero coordinate prefers +
    }
    // integer-type root: two largest |P_i| with matching signs
    int a1 = -1, a2 = -1, i1 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (w[i] > a1) { a2 = a1; a1 = w[i]; i1 = i; }
        else if (w[i] > a2) { a2 = w[i]; }
    }
    int RI[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) RI[i] = 0;
    if (a1 > a2) {
        // forced i1; the partner is the first tied index with a + sign,
        // else the last tied index
        int jpos = -1, jlast = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j != i1 && w[j] == a2) {
                if (s[j] > 0 && jpos < 0) jpos = j;
                jlast = j;
            }
        const int j = jpos >= 0 ? jpos : jlast;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i == i1) RI[i] = 2 * s[i];
            if (i == j) RI[i] = 2 * s[i];
        }
    } else {
        // choose two of the indices tied at a1: take + signs early, put
        // - signs as late as possible
        int remaining = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) remaining += (w[i] == a1) ? 1 : 0;
        int need = 2;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (w[k] == a1) {
                --remaining;
                if (need > 0 && (s[k] > 0 || remaining < need)) {
                    RI[k] = 2 * s[k];
                    --need;
                }
            }
    }
    const int vI = 2 * (a1 + a2);

    // half-type root: signs of P, with one flip if the minus count is odd
    int RH[8];
    int vH = 0, nneg = 0, zlast = -1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        RH[i] = s[i];
        vH += w[i];
        nneg += s[i] < 0 ? 1 : 0;
        if (P[i] == 0) zlast = i;
    }
    if (nneg & 1) {
        if (zlast >= 0) {
            // flipping a zero coordinate costs nothing; the last one keeps R largest
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i == zlast) RH[i] = -1;
        } else {
            int wmin = w[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) wmin = min(wmin, w[i]);
            int kneg = -1, klast = -1;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (w[k] == wmin) {
                    if (s[k] < 0 && kneg < 0) kneg = k;
                    klast = k;
                }
            const int k = kneg >= 0 ? kneg : klast;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i == k) RH[i] = -RH[i];
            vH -= 2 * wmin;
        }
    }
    // RI[0] is in {-2, 0, 2} and RH[0] in {-1, 1}: position 0 decides a tie
    const bool useI = (vI > vH) || (vI == vH && RI[0] > RH[0]);
#pragma unroll
    for (int i = 0; i < 8; ++i) R[i] = useI ? RI[i] : RH[i];
}

// bf16 nearest (ties to even) to the exact product s * q, with q a small
// integer (|q| < 2^15): the product is first rounded to fp32 by
// truncation with a sticky low bit (round to odd), which makes the later
// round-to-nearest-even to bf16 equal to one rounding of the exact value
// (24 >= 8 + 2 bits; Boldo & Melquiond, "Emulation of FMA and correctly
// rounded sums: proved algorithms using rounding to odd", 2008).
__device__ __forceinline__ __nv_bfloat16 bf16_of_product(float s, float q) {
    if (fabsf(s) < 1e-30f) {  // keep the residual test clear of underflow
        return __double2bfloat16(static_cast<double>(s) * static_cast<double>(q));
    }
    const float p = __fmul_rz(s, q);
    const float r = fmaf(s, q, -p);
    unsigned b = __float_as_uint(p);
    if (r != 0.f) b |= 1u;
    return __float2bfloat16_rn(__uint_as_float(b));
}

__device__ __forceinline__ unsigned pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return static_cast<unsigned>(__bfloat16_as_ushort(lo)) | (static_cast<unsigned>(__bfloat16_as_ushort(hi)) << 16);
}

__device__ __forceinline__ int8_t coord_of(uint2 packed, int i) {
    const unsigned w = i < 4 ? packed.x : packed.y;
    return static_cast<int8_t>((w >> (8 * (i & 3))) & 0xFF);
}

}  // namespace e8q
