// K1: randomized Hadamard transform + row scale + E8 projection + core
// encoding + ordered escape compaction (+ optional dequantised output),
// one launch over a batch of matrices ("E8-QAT", Figure 2 (a)-(c)).
//
// Work unit: a row tile (whole rows of one matrix, about 4K elements).
// Persistent CTAs take tiles from an atomic ticket; the ticket order is the
// group order, so each tile's escape / overflow records are placed by a
// decoupled look-back over the previous tiles' counts, which yields the
// records sorted by group and a CSR row index in one pass.  Every wait in
// the look-back is bounded; running out sets counters->err.
#pragma once
#include "common.cuh"
#include "lattice.cuh"

namespace e8q {

constexpr int kEncThreads = 256;
constexpr int kSpinLimit = 1 << 22;

template <int MAXM>
struct EncodeParams {
    e8q_escape* esc;
    e8q_overflow* ovf;
    int64_t* esc_rp;
    int64_t* ovf_rp;
    e8q_counters* ctr;
    unsigned long long* ws;  // [0] tile ticket, [1] unused, [2 + t] tile status
    long long esc_cap;
    long long ovf_cap;
    float kappa;
    int32_t dq_mode;
    int32_t scale_in;
    int32_t n_mats;
    int32_t n_tiles;
    int32_t total_rows;
    int32_t clamp;      // fast kernel: inputs may reach |2x| >= 2^14 (given scales or large kappa)
    int32_t core_only;   // the core-clipped projection (E8Q_ENCODE_CORE_ONLY)
    int32_t shape_gain;  // the shape-gain code (E8Q_ENCODE_SHAPE_GAIN)
    MatDesc m[MAXM];
};

// Shape-gain code of X = 2x (sg_code in lattice.cuh), out of line for the
// general kernel.
__device__ __noinline__ int shape_gain_code(const float (&X)[8], int (&P)[8], float* xm, const uint16_t* __restrict__ st1,
                                            const uint16_t* __restrict__ st2) {
    return sg_code(X, P, *xm, st1, st2);
}

// Nearest core point of X = 2x whose nearest E8 point P lies outside the
// core ("E8-QAT", Figure 2 (a): post-training quantisation starts from the
// fixed core).  Equal distances go to the smaller core index.  On return P
// holds the core point; the result is its core index.
//
// A first bound comes from two points near x: the escape base P - r (the
// escape rule's root), when in the core, and the nearest E8 point of x
// pulled in to |x|^2 = 6, which is always in the core.  Then every E8 point
// c within that distance of x and with |c|^2 <= 12 (a superset of the core)
// is visited by a depth-first enumeration of each coset (D8 and D8 + 1/2:
// integer vectors z, or z + 1/2, with an even coordinate sum), the radius
// shrinking as closer core points are found; each point visited is checked
// against the core by its rank.
__device__ __noinline__ int nearest_core_point(const float (&X)[8], int (&P)[8], const uint16_t* __restrict__ st1,
                                               const uint16_t* __restrict__ st2) {
    float best = INFINITY;  // squared distance, x units
    int brank = 0x7FFFFFFF;
    int bP[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) bP[i] = 0;
    auto consider = [&](const int (&C)[8]) {
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float t = 0.5f * (X[i] - static_cast<float>(C[i]));
            d = fmaf(t, t, d);
        }
        if (d <= best) {
            const int r = core_rank(C, st1, st2);
            if (r >= 0 && (d < best || r < brank)) {
                best = d;
                brank = r;
#pragma unroll
                for (int i = 0; i < 8; ++i) bP[i] = C[i];
            }
        }
    };
    {
        int R[8], Q[8];
        best_escape_root(P, R);
#pragma unroll
        for (int i = 0; i < 8; ++i) Q[i] = P[i] - R[i];
        consider(Q);
        // x pulled in to |x'|^2 = 6: its nearest E8 point p' has |p'| <= sqrt(6) + 1
        // (the covering radius is 1), so |p'|^2 <= 10 and p' is in the core
        float n2 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) n2 = fmaf(X[i], X[i], n2);
        const float k = fminf(4.8989795f * rsqrtf(fmaxf(n2, 1e-30f)), 1.f);  // |2x'| = 2 sqrt(6)
        float Xs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) Xs[i] = X[i] * k;
        int Ps[8];
        e8_nearest_doubled(Xs, Ps);
        consider(Ps);
    }
    // every E8 point c within the current distance of x with |c|^2 <= 12 (all
    // core points have), coset by coset, depth first over the coordinates
    constexpr float kCoreN2 = 12.f + 1e-3f;
    for (int coset = 0; coset < 2; ++coset) {
        const float off = coset ? 0.5f : 0.f;
        float cy[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cy[i] = 0.5f * X[i] - off;
        int z[8], hi[8];
        float part[9], pn[9];  // partial squared distance to x, partial squared norm of c
        part[0] = 0.f;
        pn[0] = 0.f;
        int lvl = 0;
        auto bounds = [&](int l) {
            const float sq = sqrtf(fmaxf(best - part[l], 0.f));
            const float sn = sqrtf(fmaxf(kCoreN2 - pn[l], 0.f));
            z[l] = max(static_cast<int>(ceilf(cy[l] - sq)), static_cast<int>(ceilf(-sn - off)));
            hi[l] = min(static_cast<int>(floorf(cy[l] + sq)), static_cast<int>(floorf(sn - off)));
        };
        bounds(0);
        int guard = 0;
        while (lvl >= 0 && ++guard < (1 << 22)) {  // bounded: the lens holds at most the 117,361 points of |c|^2 <= 12
            if (z[lvl] > hi[lvl]) {
                --lvl;
                if (lvl >= 0) ++z[lvl];
                continue;
            }
            const float t = cy[lvl] - static_cast<float>(z[lvl]);
            const float pt = fmaf(t, t, part[lvl]);
            const float c = static_cast<float>(z[lvl]) + off;
            const float pc = fmaf(c, c, pn[lvl]);
            if (pt > best || pc > kCoreN2) {
                ++z[lvl];
                continue;
            }
            if (lvl == 7) {
                int sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) sum += z[i];
                if ((sum & 1) == 0) {
                    int C[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) C[i] = 2 * z[i] + coset;
                    consider(C);
                }
                ++z[lvl];
                continue;
            }
            part[lvl + 1] = pt;
            pn[lvl + 1] = pc;
            ++lvl;
            bounds(lvl);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = bP[i];
    return brank == 0x7FFFFFFF ? 0 : brank;
}

// shared-memory layout of the encode kernel (bytes)
constexpr int kEncTileBytes = kTileMaxElems * 4;                      // 65536
constexpr int kEncT1Bytes = ((2 * 2401 * 7 * 2 + 15) / 16) * 16;     // 67232
constexpr int kEncT2Bytes = ((2 * 2401 * 2 + 15) / 16) * 16;         // 9616
constexpr int kEncEscBytes = kTileMaxGroups * 8;                      // 16384
constexpr int kEncOvfBytes = kTileMaxGroups * 20;                     // 40960
constexpr int kEncSmemBytes = kEncTileBytes + kEncT1Bytes + kEncT2Bytes + kEncEscBytes + kEncOvfBytes;

template <int MAXM>
__device__ __forceinline__ int find_matrix(const EncodeParams<MAXM>& p, int t) {
    int lo = 0, hi = p.n_mats - 1;
    while (lo < hi) {  // last matrix whose tile_base <= t
        const int mid = (lo + hi + 1) >> 1;
        if (p.m[mid].tile_base <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Place this tile's records after all earlier tiles' ones.  Warp 0 only.
// Status word: bits 62..63 flag (1 aggregate, 2 inclusive prefix), bits
// 31..61 escape count, bits 0..30 overflow count.
__device__ inline void lookback(unsigned long long* status, int t, unsigned ne, unsigned no, unsigned& ex_e,
                                unsigned& ex_o, unsigned long long* err) {
    const unsigned long long kAgg = 1ull << 62, kPre = 2ull << 62;
    const int lane = threadIdx.x & 31;
    const unsigned long long own = (static_cast<unsigned long long>(ne) << 31) | no;
    if (lane == 0) st_volatile_u64(&status[t], (t == 0 ? kPre : kAgg) | own);
    unsigned acc_e = 0, acc_o = 0;
    if (t > 0) {
        int j = t - 1;
        int spins = 0;
        while (true) {
            const int k = j - lane;
            const unsigned long long s = (k >= 0) ? ld_volatile_u64(&status[k]) : kPre;
            const unsigned flag = static_cast<unsigned>(s >> 62);
            const unsigned notready = __ballot_sync(0xFFFFFFFFu, flag == 0);
            const unsigned ispre = __ballot_sync(0xFFFFFFFFu, flag == 2);
            const unsigned window = ispre ? (((ispre & (0u - ispre)) << 1) - 1u) : 0xFFFFFFFFu;
            if (notready & window) {
                if (++spins > kSpinLimit) {
                    if (lane == 0) atomicOr(err, 1ull);
                    break;
                }
                __nanosleep(64);
                continue;
            }
            const bool in = (window >> lane) & 1u;
            unsigned ve = in ? static_cast<unsigned>((s >> 31) & 0x7FFFFFFFu) : 0u;
            unsigned vo = in ? static_cast<unsigned>(s & 0x7FFFFFFFu) : 0u;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                ve += __shfl_xor_sync(0xFFFFFFFFu, ve, off);
                vo += __shfl_xor_sync(0xFFFFFFFFu, vo, off);
            }
            acc_e += ve;
            acc_o += vo;
            if (ispre) break;
            j -= 32;
        }
        if (lane == 0)
            st_volatile_u64(&status[t],
                            kPre | (static_cast<unsigned long long>((acc_e + ne) & 0x7FFFFFFFu) << 31) |
                                ((acc_o + no) & 0x7FFFFFFFu));
    }
    ex_e = acc_e;
    ex_o = acc_o;
}

template <int MAXM>
__global__ void __launch_bounds__(kEncThreads, 1) k_encode(const __grid_constant__ EncodeParams<MAXM> p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* tile = reinterpret_cast<float*>(smem);
    uint16_t* st1 = reinterpret_cast<uint16_t*>(smem + kEncTileBytes);
    uint16_t* st2 = reinterpret_cast<uint16_t*>(smem + kEncTileBytes + kEncT1Bytes);
    e8q_escape* esc_st = reinterpret_cast<e8q_escape*>(smem + kEncTileBytes + kEncT1Bytes + kEncT2Bytes);
    e8q_overflow* ovf_st =
        reinterpret_cast<e8q_overflow*>(smem + kEncTileBytes + kEncT1Bytes + kEncT2Bytes + kEncEscBytes);

    __shared__ float s_rowc[kMaxTileRows];   // multiplier giving doubled coordinates
    __shared__ float s_rows[kMaxTileRows];   // the row scale
    __shared__ int s_eoff[kMaxTileRows + 1];
    __shared__ int s_ooff[kMaxTileRows + 1];
    __shared__ float s_part[kEncThreads / 32];
    __shared__ int s_wc[2 * (kEncThreads / 32)];
    __shared__ int s_ticket;
    __shared__ unsigned s_ex[2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kEncThreads / 32;

    // constant tables into shared memory
    {
        const uint4* a = reinterpret_cast<const uint4*>(g_t1);
        uint4* b = reinterpret_cast<uint4*>(st1);
        for (int i = tid; i < (2 * 2401 * 7 * 2) / 16; i += kEncThreads) b[i] = a[i];
        for (int i = ((2 * 2401 * 7 * 2) / 16) * 8 + tid; i < 2 * 2401 * 7; i += kEncThreads) st1[i] = g_t1[i];
        for (int i = tid; i < 2 * 2401; i += kEncThreads) st2[i] = g_t2[i];
    }
    unsigned long long nonfinite = 0, clamped = 0;

    for (;;) {
        if (tid == 0) s_ticket = static_cast<int>(atomicAdd(&p.ws[0], 1ull));
        __syncthreads();
        const int t = s_ticket;
        if (t >= p.n_tiles) break;
        const MatDesc& M = p.m[find_matrix(p, t)];
        const int C = M.cols, gpr = C >> 3;
        const int rpt = meta_rpt(M.meta), logb = meta_logb(M.meta);
        const int r0 = (t - M.tile_base) * rpt;
        const int nr = min(rpt, M.rows - r0);
        const int n = nr * C, G = nr * gpr;
        const float B = static_cast<float>(1 << logb);

        // 1. load, sign flip, non-finite -> 0
        if (meta_bf16(M.meta)) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(M.w) + static_cast<size_t>(r0) * C);
            for (int q = tid; q < (n >> 3); q += kEncThreads) {
                const uint4 raw = __ldcs(src + q);
                const int c0 = (q << 3) % C;
                const uint2 dv = *reinterpret_cast<const uint2*>(M.signs + c0);
                const unsigned wv[4] = {raw.x, raw.y, raw.z, raw.w};
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float x = __uint_as_float((i & 1) ? (wv[i >> 1] & 0xFFFF0000u) : (wv[i >> 1] << 16));
                    if (!isfinite(x)) { x = 0.f; ++nonfinite; }
                    const int8_t sg = static_cast<int8_t>(((i < 4 ? dv.x : dv.y) >> (8 * (i & 3))) & 0xFF);
                    f[i] = sg < 0 ? -x : x;
                }
                float4* dst = reinterpret_cast<float4*>(tile + (q << 3));
                dst[0] = make_float4(f[0], f[1], f[2], f[3]);
                dst[1] = make_float4(f[4], f[5], f[6], f[7]);
            }
        } else {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(M.w) + static_cast<size_t>(r0) * C);
            for (int q = tid; q < (n >> 2); q += kEncThreads) {
                const float4 raw = __ldcs(src + q);
                const int c0 = (q << 2) % C;
                const unsigned dv = *reinterpret_cast<const unsigned*>(M.signs + c0);
                float f[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (!isfinite(f[i])) { f[i] = 0.f; ++nonfinite; }
                    const int8_t sg = static_cast<int8_t>((dv >> (8 * i)) & 0xFF);
                    f[i] = sg < 0 ? -f[i] : f[i];
                }
                reinterpret_cast<float4*>(tile)[q] = make_float4(f[0], f[1], f[2], f[3]);
            }
        }
        __syncthreads();

        // 2. unnormalised blockwise Hadamard
        if (logb > 0) fwht_smem(tile, n, logb);

        // 3. row sums of squares -> scale and multiplier (deterministic tree)
        {
            int nrp = 1;
            while (nrp < nr) nrp <<= 1;
            const int tpr = kEncThreads / nrp;
            const int r = tid / tpr, j = tid % tpr;
            float acc = 0.f;
            if (r < nr)
                for (int c = j; c < C; c += tpr) {
                    const float v = tile[r * C + c];
                    acc = fmaf(v, v, acc);
                }
            if (tpr <= 32) {
                for (int off = tpr >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
                if (j == 0 && r < nr) s_rows[r] = acc;  // raw sum for now
            } else {
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
                if (lane == 0) s_part[warp] = acc;
            }
            __syncthreads();
            if (tpr > 32 && j == 0 && r < nr) {
                float a = 0.f;
                for (int w = 0; w < tpr / 32; ++w) a += s_part[r * (tpr / 32) + w];
                s_rows[r] = a;
            }
            __syncthreads();
            if (tid < nr) {
                float s;
                if (p.scale_in) {
                    s = M.scale[r0 + tid];
                    if (!(s > 0.f) || !isfinite(s)) s = 0.f;
                } else {
                    s = sqrtf(s_rows[tid] / (B * static_cast<float>(C))) / p.kappa;
                    M.scale[r0 + tid] = s;
                }
                s_rows[tid] = s;
                s_rowc[tid] = (s > 0.f) ? 2.0f / (s * sqrtf(B)) : 0.f;
            }
            __syncthreads();
        }

        // 4. project, encode, stage records in group order
        unsigned ne = 0, no = 0;
        const size_t gbase_local = static_cast<size_t>(r0) * gpr;
        for (int base = 0; base < G; base += kEncThreads) {
            const int g = base + tid;
            int kind = 0, idxv = 0, rootv = 0;
            int P[8];
            float xm = 0.5f;  // x-hat = xm P: the lattice point p = P / 2, or the shape-gain reconstruction
            if (g < G) {
                const int r = g / gpr;
                const float c = s_rowc[r];
                const float4 v0 = reinterpret_cast<const float4*>(tile)[2 * g];
                const float4 v1 = reinterpret_cast<const float4*>(tile)[2 * g + 1];
                const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                float X[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) X[i] = fminf(fmaxf(fmaf(vv[i], c, 0.f), -1048576.f), 1048576.f);
                if (p.shape_gain) {
                    idxv = shape_gain_code(X, P, &xm, st1, st2);
                } else {
                    e8_nearest_doubled(X, P);
                    const int rk = core_rank(P, st1, st2);
                    if (rk >= 0) {
                        idxv = rk;
                    } else if (p.core_only) {
                        idxv = nearest_core_point(X, P, st1, st2);
                    } else {
                        int R[8], Q[8];
                        best_escape_root(P, R);
#pragma unroll
                        for (int i = 0; i < 8; ++i) Q[i] = P[i] - R[i];
                        const int rq = core_rank(Q, st1, st2);
                        if (rq >= 0) {
                            kind = 1;
                            idxv = rq;
                            rootv = core_rank(R, st1, st2) - 1;
                        } else {
                            kind = 2;
                        }
                    }
                }
                M.idx[gbase_local + g] = static_cast<uint16_t>(idxv);
                if (p.dq_mode == E8Q_DEQUANT_ROTATED) {
                    const float s = s_rows[r];
                    uint4 o;
                    o.x = pack_bf16x2(bf16_of_product(s, xm * P[0]), bf16_of_product(s, xm * P[1]));
                    o.y = pack_bf16x2(bf16_of_product(s, xm * P[2]), bf16_of_product(s, xm * P[3]));
                    o.z = pack_bf16x2(bf16_of_product(s, xm * P[4]), bf16_of_product(s, xm * P[5]));
                    o.w = pack_bf16x2(bf16_of_product(s, xm * P[6]), bf16_of_product(s, xm * P[7]));
                    reinterpret_cast<uint4*>(static_cast<uint16_t*>(M.dq) + static_cast<size_t>(r0) * C)[g] = o;
                } else if (p.dq_mode == E8Q_DEQUANT_ORIGINAL) {
                    // x-hat itself (p, or the shape-gain reconstruction); H of it stays
                    // exact in fp32 and is scaled once afterwards
                    float4* dst = reinterpret_cast<float4*>(tile) + 2 * g;
                    dst[0] = make_float4(xm * P[0], xm * P[1], xm * P[2], xm * P[3]);
                    dst[1] = make_float4(xm * P[4], xm * P[5], xm * P[6], xm * P[7]);
                }
            }
            const unsigned be = __ballot_sync(0xFFFFFFFFu, kind == 1);
            const unsigned bo = __ballot_sync(0xFFFFFFFFu, kind == 2);
            if (lane == 0) {
                s_wc[warp] = __popc(be);
                s_wc[kWarps + warp] = __popc(bo);
            }
            __syncthreads();
            unsigned pe = ne, po = no, te = 0, to = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                if (w < warp) { pe += s_wc[w]; po += s_wc[kWarps + w]; }
                te += s_wc[w];
                to += s_wc[kWarps + w];
            }
            const uint32_t gid = M.group_base + static_cast<uint32_t>(gbase_local + g);
            if (kind == 1) {
                e8q_escape rec;
                rec.group = gid;
                rec.core = static_cast<uint16_t>(idxv);
                rec.root = static_cast<uint8_t>(rootv);
                rec.reserved = 0;
                esc_st[pe + __popc(be & lanemask_lt())] = rec;
            } else if (kind == 2) {
                e8q_overflow rec;
                rec.group = gid;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    int v = P[i];
                    if (v > 32767 || v < -32768) { ++clamped; v = v > 0 ? 32767 : -32768; }
                    rec.coord2[i] = static_cast<int16_t>(v);
                }
                ovf_st[po + __popc(bo & lanemask_lt())] = rec;
            }
            ne += te;
            no += to;
            __syncthreads();
        }

        // per-row offsets inside the tile (records are sorted by group)
        if (tid <= nr) {
            const uint32_t lim = M.group_base + static_cast<uint32_t>(gbase_local + static_cast<size_t>(tid) * gpr);
            int lo = 0, hi = static_cast<int>(ne);
            while (lo < hi) { const int mid = (lo + hi) >> 1; if (esc_st[mid].group < lim) lo = mid + 1; else hi = mid; }
            s_eoff[tid] = lo;
            lo = 0; hi = static_cast<int>(no);
            while (lo < hi) { const int mid = (lo + hi) >> 1; if (ovf_st[mid].group < lim) lo = mid + 1; else hi = mid; }
            s_ooff[tid] = lo;
        }

        // 5. original-basis dequant: inverse transform of s * p in place
        if (p.dq_mode == E8Q_DEQUANT_ORIGINAL) {
            __syncthreads();
            if (logb > 0) fwht_smem(tile, n, logb);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(M.dq) + static_cast<size_t>(r0) * C);
            for (int q = tid; q < (n >> 3); q += kEncThreads) {
                const int c0 = (q << 3) % C;
                const float inv = s_rows[(q << 3) / C] / sqrtf(B);
                const uint2 dv = *reinterpret_cast<const uint2*>(M.signs + c0);
                const float4 a = reinterpret_cast<const float4*>(tile)[2 * q];
                const float4 b = reinterpret_cast<const float4*>(tile)[2 * q + 1];
                const float vv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                __nv_bfloat16 o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int8_t sg = static_cast<int8_t>(((i < 4 ? dv.x : dv.y) >> (8 * (i & 3))) & 0xFF);
                    const float y = vv[i] * inv;
                    o[i] = __float2bfloat16_rn(sg < 0 ? -y : y);
                }
                dst[q] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                    pack_bf16x2(o[6], o[7]));
            }
        }

        // 6. place the tile's records after the earlier tiles' ones
        __syncthreads();
        if (warp == 0) {
            unsigned ex_e, ex_o;
            lookback(p.ws + 2, t, ne, no, ex_e, ex_o, &p.ctr->err);
            if (lane == 0) { s_ex[0] = ex_e; s_ex[1] = ex_o; }
        }
        __syncthreads();
        const long long ex_e = s_ex[0], ex_o = s_ex[1];
        if (tid < nr) {
            if (p.esc_rp) p.esc_rp[M.row_base + r0 + tid] = ex_e + s_eoff[tid];
            if (p.ovf_rp) p.ovf_rp[M.row_base + r0 + tid] = ex_o + s_ooff[tid];
        }
        if (t == p.n_tiles - 1 && tid == 0) {
            const long long te = ex_e + ne, to = ex_o + no;
            if (p.esc_rp) p.esc_rp[p.total_rows] = te;
            if (p.ovf_rp) p.ovf_rp[p.total_rows] = to;
            p.ctr->n_escape = te;
            p.ctr->n_overflow = to;
            p.ctr->n_dropped = (te > p.esc_cap ? te - p.esc_cap : 0) + (to > p.ovf_cap ? to - p.ovf_cap : 0);
        }
        for (int i = tid; i < static_cast<int>(ne); i += kEncThreads) {
            const long long pos = ex_e + i;
            if (pos < p.esc_cap) p.esc[pos] = esc_st[i];
        }
        for (int i = tid; i < static_cast<int>(no); i += kEncThreads) {
            const long long pos = ex_o + i;
            if (pos < p.ovf_cap) p.ovf[pos] = ovf_st[i];
        }
        __syncthreads();
    }

    // counters that every CTA contributes to
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        nonfinite += __shfl_xor_sync(0xFFFFFFFFu, nonfinite, off);
        clamped += __shfl_xor_sync(0xFFFFFFFFu, clamped, off);
    }
    if (lane == 0) {
        if (nonfinite) atomicAdd(&p.ctr->n_nonfinite, nonfinite);
        if (clamped) atomicAdd(&p.ctr->n_clamped, clamped);
    }
}

}  // namespace e8q
