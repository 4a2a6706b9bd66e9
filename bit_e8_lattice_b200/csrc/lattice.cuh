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

// bf16 nearest of the exact products s * P0 / 2 and s * P1 / 2 (P small
// integers, |P| < 2^16), packed lo | hi << 16: the same round-to-odd
// argument as bf16_of_product on fp32 pairs.  s / 2 is exact for
// |s| >= 1e-30; smaller scales take the double product.
__device__ __forceinline__ unsigned bf16x2_of_half_products(float s, float P0, float P1) {
    if (fabsf(s) < 1e-30f) {
        const double sd = 0.5 * static_cast<double>(s);
        return pack_bf16x2(__double2bfloat16(sd * static_cast<double>(P0)), __double2bfloat16(sd * static_cast<double>(P1)));
    }
    const float sh = 0.5f * s;
    const float2 q = make_float2(P0, P1), ss = make_float2(sh, sh);
    const float2 p = __fmul2_rz(ss, q);
    const float2 r = __ffma2_rn(ss, q, make_float2(-p.x, -p.y));
    const float lo = __uint_as_float(__float_as_uint(p.x) | (r.x != 0.f ? 1u : 0u));
    const float hi = __uint_as_float(__float_as_uint(p.y) | (r.y != 0.f ? 1u : 0u));
    const __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const unsigned*>(&t);
}

// The 8 signed bytes of a packed point as exact floats: each byte, biased by
// 128, is placed under the exponent of 2^23 and the bias removed again.
__device__ __forceinline__ void bytes_to_floats(uint2 w, float (&f)[8]) {
    const unsigned x = w.x ^ 0x80808080u, y = w.y ^ 0x80808080u;
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
        const float2 a = make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440u + j)),
                                     __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441u + j)));
        const float2 b = make_float2(__uint_as_float(__byte_perm(y, 0x4B000000u, 0x7440u + j)),
                                     __uint_as_float(__byte_perm(y, 0x4B000000u, 0x7441u + j)));
        const float2 fa = __fadd2_rn(a, make_float2(-8388736.f, -8388736.f));
        const float2 fb = __fadd2_rn(b, make_float2(-8388736.f, -8388736.f));
        f[j] = fa.x;
        f[j + 1] = fa.y;
        f[4 + j] = fb.x;
        f[4 + j + 1] = fb.y;
    }
}

__device__ __forceinline__ int8_t coord_of(uint2 packed, int i) {
    const unsigned w = i < 4 ? packed.x : packed.y;
    return static_cast<int8_t>((w >> (8 * (i & 3))) & 0xFF);
}

}  // namespace e8q

namespace e8q {

// Same nearest point as e8_nearest_doubled, with fewer instructions: packed
// fp32 pairs for the rounding, parities from the xor of raw bits, and the
// parity fix applied to the first coordinate whose error equals the extreme
// one (no index tracking).  Returns the lattice point as exact floats P
// (doubled coordinates) and whether it is of the odd (D8 + 1/2) type.
__device__ __forceinline__ bool e8_nearest_lean(const float (&X)[8], float (&P)[8]) {
    const float kM = 25165824.0f;  // 1.5 * 2^24
    float E[8], e[8];
    unsigned gx = 0u, ex = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 x = make_float2(X[2 * j], X[2 * j + 1]);
        const float2 g = __fadd2_rn(x, make_float2(kM, kM));
        const float2 Ev = __fadd2_rn(g, make_float2(-kM, -kM));
        const float2 d = __ffma2_rn(Ev, make_float2(-1.f, -1.f), x);
        gx ^= __float_as_uint(g.x) ^ __float_as_uint(g.y);
        ex ^= __float_as_uint(d.x) ^ __float_as_uint(d.y);
        E[2 * j] = Ev.x; E[2 * j + 1] = Ev.y;
        e[2 * j] = d.x; e[2 * j + 1] = d.y;
    }
    const bool oddA = (gx & 1u) != 0;              // sum of E/2 is odd
    const bool oddB = ((gx ^ (ex >> 31)) & 1u) != 0;  // parity of sum(E/2) differs from that of the minus count
    float2 q = __fmul2_rn(make_float2(e[0], e[1]), make_float2(e[0], e[1]));
    q = __ffma2_rn(make_float2(e[2], e[3]), make_float2(e[2], e[3]), q);
    q = __ffma2_rn(make_float2(e[4], e[5]), make_float2(e[4], e[5]), q);
    q = __ffma2_rn(make_float2(e[6], e[7]), make_float2(e[6], e[7]), q);
    const float da = q.x + q.y;
    const float st = ((fabsf(e[0]) + fabsf(e[1])) + (fabsf(e[2]) + fabsf(e[3]))) +
                     ((fabsf(e[4]) + fabsf(e[5])) + (fabsf(e[6]) + fabsf(e[7])));
    const float tmax = fmaxf(fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3]))),
                             fmaxf(fmaxf(fabsf(e[4]), fabsf(e[5])), fmaxf(fabsf(e[6]), fabsf(e[7]))));
    const float tmin = fminf(fminf(fminf(fabsf(e[0]), fabsf(e[1])), fminf(fabsf(e[2]), fabsf(e[3]))),
                             fminf(fminf(fabsf(e[4]), fabsf(e[5])), fminf(fabsf(e[6]), fabsf(e[7]))));
    const float DA = da + (oddA ? (4.f - 4.f * tmax) : 0.f);
    const float DB = (8.f - 2.f * st + da) + (oddB ? 4.f * tmin : 0.f);
    const bool useB = DB < DA;
    const float ub = useB ? 1.f : 0.f;
    const float m = useB ? tmin : tmax;
    const float dir = useB ? -2.f : 2.f;  // towards x: the error's sign (D8), its opposite (D8 + 1/2)
    bool pending = useB ? oddB : oddA;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float sg = __uint_as_float((__float_as_uint(e[i]) & 0x80000000u) | 0x3F800000u);
        float p = fmaf(sg, ub, E[i]);
        const bool hit = pending && fabsf(e[i]) == m;
        pending = pending && !hit;
        p = hit ? fmaf(sg, dir, p) : p;
        P[i] = p;
    }
    return useB;
}

// Shape-gain code of X = 2x (SQuAT page, "shape and scale split": a unit
// direction quantised against a spherical E8 codebook, a scalar gain
// through a low-bit scalar quantiser).  Directions: the 2160 points of the
// |p|^2 = 4 shell, core indices kSgShellFirst .. + 2159; the best is the one
// of largest <X, P>, taken per family of the shell (doubled coordinates):
//   +-4 e_i                       4 max |X_i|
//   +-2 on four coordinates       2 (sum of the four largest |X_i|)
//   odd, one +-3, sum = 0 mod 4   sum |X_i| + 2 |X_j| for the +-3 at j, less
//                                 the cheapest sign reversal when the number
//                                 of negative X_i is even (the sum rule):
//                                 2 |X_i| for a +-1, 6 |X_j| for the +-3.
// Gain level k = min(15, floor(|x| / (6 / 16))).  On return P holds the
// direction's doubled point and xm the factor (k + 1/2) (6 / 16) / 4 that
// maps P to the reconstruction x-hat = xm P; the result is k << 12 | the
// direction's index in the shell.
constexpr int kSgShellFirst = 241;
constexpr float kSgStep = 6.0f / 16.0f;

__device__ __forceinline__ int sg_code(const float (&X)[8], int (&P)[8], float& xm, const uint16_t* __restrict__ st1,
                                       const uint16_t* __restrict__ st2) {
    float a[8];
    float n2 = 0.f, total = 0.f;
    int neg = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[i] = fabsf(X[i]);
        n2 = fmaf(X[i], X[i], n2);
        total += a[i];
        neg += X[i] < 0.f;
    }
    // family +-4 e_i; the four largest |X_i| (rank by value, then position);
    // the two smallest
    int imax = 0, imin = 0, imin2 = -1;
    float top4 = 0.f;
    unsigned in4 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (a[i] > a[imax]) imax = i;
        int r = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) r += (a[k] > a[i]) || (a[k] == a[i] && k < i);
        if (r < 4) {
            top4 += a[i];
            in4 |= 1u << i;
        }
        if (a[i] < a[imin]) imin = i;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i != imin && (imin2 < 0 || a[i] < a[imin2])) imin2 = i;
    const float sA = 4.f * a[imax], sB = 2.f * top4;
    // odd family: the +-3 at j
    float sC = -INFINITY;
    int jC = 0, fC = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float sc = total + 2.f * a[j];
        int f = -1;
        if ((neg & 1) == 0) {
            const int o = (j == imin) ? imin2 : imin;  // smallest |X_i|, i != j
            const float c1 = 2.f * a[o], c3 = 6.f * a[j];
            if (c3 < c1) {
                sc -= c3;
                f = j;
            } else {
                sc -= c1;
                f = o;
            }
        }
        if (sc > sC) {
            sC = sc;
            jC = j;
            fC = f;
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int sg = X[i] < 0.f ? -1 : 1;
        if (sA >= sB && sA >= sC) {
            P[i] = i == imax ? 4 * sg : 0;
        } else if (sB >= sC) {
            P[i] = ((in4 >> i) & 1u) ? 2 * sg : 0;
        } else {
            const int v = (i == jC ? 3 : 1) * sg;
            P[i] = i == fC ? -v : v;
        }
    }
    const float g = 0.5f * sqrtf(n2);
    const int k = min(15, static_cast<int>(floorf(g / kSgStep)));
    xm = (static_cast<float>(k) + 0.5f) * kSgStep * 0.25f;
    return (k << 12) | (core_rank(P, st1, st2) - kSgShellFirst);
}

// Core index of a point given as exact floats (doubled coordinates) and its
// type, or -1 outside the core; the two table keys are formed with exact
// small-integer float arithmetic.
__device__ __forceinline__ int core_rank_f(const float (&P)[8], bool odd, const uint16_t* __restrict__ t1,
                                           const uint16_t* __restrict__ t2) {
    float2 n = __fmul2_rn(make_float2(P[0], P[4]), make_float2(P[0], P[4]));
    n = __ffma2_rn(make_float2(P[1], P[5]), make_float2(P[1], P[5]), n);
    n = __ffma2_rn(make_float2(P[2], P[6]), make_float2(P[2], P[6]), n);
    n = __ffma2_rn(make_float2(P[3], P[7]), make_float2(P[3], P[7]), n);
    const float n2 = n.x + n.y;
    if (!(n2 <= 48.f)) return -1;
    float2 k = __fmul2_rn(make_float2(P[0], P[4]), make_float2(343.f, 343.f));
    k = __ffma2_rn(make_float2(P[1], P[5]), make_float2(49.f, 49.f), k);
    k = __ffma2_rn(make_float2(P[2], P[6]), make_float2(7.f, 7.f), k);
    k = __fadd2_rn(make_float2(P[3], P[7]), k);
    // base-7 digits (P + 6) >> 1, plus 2401 for the odd type
    const float base = odd ? 3401.f : 1200.f;  // even digit (P + 6) / 2: 0.5 k + 1200; odd (P + 5) / 2: 0.5 k + 1000
    const float hk = fmaf(k.x, 0.5f, base), lk = fmaf(k.y, 0.5f, base);
    const float i1 = fmaf(hk, 7.f, n2 * 0.125f);
    const int a = t1[__float_as_int(i1 + 8388608.f) - 0x4B000000];
    const int b = t2[__float_as_int(lk + 8388608.f) - 0x4B000000];
    const int r = a + b;
    return (a != 0xFFFF && r < 65536) ? r : -1;
}

// core_rank_f without a branch, given n2 = |P|^2: both table reads happen
// for every group (index 0 outside the key range), so that a warp's groups
// stay converged.
__device__ __forceinline__ int core_rank_nb(const float (&P)[8], bool odd, float n2, const uint16_t* __restrict__ t1,
                                            const uint16_t* __restrict__ t2) {
    const bool inr = n2 <= 48.f;  // then every |P_i| <= 6: digits in 0..6
    float2 k = __fmul2_rn(make_float2(P[0], P[4]), make_float2(343.f, 343.f));
    k = __ffma2_rn(make_float2(P[1], P[5]), make_float2(49.f, 49.f), k);
    k = __ffma2_rn(make_float2(P[2], P[6]), make_float2(7.f, 7.f), k);
    k = __fadd2_rn(make_float2(P[3], P[7]), k);
    const float base = odd ? 3401.f : 1200.f;
    const float hk = fmaf(k.x, 0.5f, base), lk = fmaf(k.y, 0.5f, base);
    const float i1 = fmaf(hk, 7.f, n2 * 0.125f);
    const int j1 = inr ? __float_as_int(i1 + 8388608.f) - 0x4B000000 : 0;
    const int j2 = inr ? __float_as_int(lk + 8388608.f) - 0x4B000000 : 0;
    const int a = t1[j1];
    const int b = t2[j2];
    const int r = a + b;
    return (inr && a != 0xFFFF && r < 65536) ? r : -1;
}

// best_escape_root with bit masks instead of index loops (same choice).
__device__ __forceinline__ void best_escape_root_lean(const int (&P)[8], int (&R)[8]) {
    int w[8];
    unsigned pos = 0u, zer = 0u, negm = 0u;
    int a1 = 0, vH = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w[i] = abs(P[i]);
        a1 = max(a1, w[i]);
        vH += w[i];
        pos |= (P[i] >= 0 ? 1u : 0u) << i;
        zer |= (P[i] == 0 ? 1u : 0u) << i;
    }
    negm = ~pos & 0xFFu;
    unsigned m1 = 0u;
    int a2 = -1, wmin = w[0];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        m1 |= (w[i] == a1 ? 1u : 0u) << i;
        a2 = max(a2, w[i] == a1 ? -1 : w[i]);
        wmin = min(wmin, w[i]);
    }
    const bool single = __popc(m1) == 1;
    if (!single) a2 = a1;
    unsigned pick;  // the two positions of the integer-type root
    if (single) {
        unsigned m2 = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) m2 |= (w[i] == a2 ? 1u : 0u) << i;
        const unsigned mp = m2 & pos;
        const unsigned j = mp ? (mp & (0u - mp)) : (1u << (31 - __clz(m2)));
        pick = m1 | j;
    } else {
        const unsigned jp = m1 & pos, jn = m1 & negm;
        const int np = __popc(jp);
        if (np >= 2) {
            const unsigned f = jp & (0u - jp);
            const unsigned r = jp & ~f;
            pick = f | (r & (0u - r));
        } else if (np == 1) {
            pick = jp | (1u << (31 - __clz(jn)));
        } else {
            const unsigned l = 1u << (31 - __clz(jn));
            const unsigned r = jn & ~l;
            pick = l | (1u << (31 - __clz(r)));
        }
    }
    const int vI = 2 * (a1 + a2);
    // half-type root: the signs of P, one flip if the minus count is odd
    unsigned hneg = negm;
    if (__popc(negm) & 1) {
        if (zer) {
            hneg |= 1u << (31 - __clz(zer));
        } else {
            unsigned T = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) T |= (w[i] == wmin ? 1u : 0u) << i;
            const unsigned tn = T & negm;
            const unsigned k = tn ? (tn & (0u - tn)) : (1u << (31 - __clz(T)));
            hneg ^= k;
            vH -= 2 * wmin;
        }
    }
    const int ri0 = (pick & 1u) ? ((pos & 1u) ? 2 : -2) : 0;
    const int rh0 = (hneg & 1u) ? -1 : 1;
    const bool useI = (vI > vH) || (vI == vH && ri0 > rh0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int ri = ((pick >> i) & 1u) ? (((pos >> i) & 1u) ? 2 : -2) : 0;
        const int rh = ((hneg >> i) & 1u) ? -1 : 1;
        R[i] = useI ? ri : rh;
    }
}

}  // namespace e8q

namespace e8q {

// core_rank with |Q|^2 supplied by the caller
__device__ __forceinline__ int core_rank_n2(const int (&P)[8], int n2, const uint16_t* __restrict__ t1,
                                            const uint16_t* __restrict__ t2) {
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

}  // namespace e8q
