// K4 + K5: dequant-GEMV from the 2-bit form ("E8-QAT", abstract: decoding
// throughput of the 2-bit representation).
//
//   y[b][r] = s_r / 2 * sum_g < P_rg , xr_b[8g .. 8g+7] >,
//   xr_b   = H_B (d (.) x_b) / sqrt(B)          (blockwise),
//   P_rg   = core[idx_rg] (+ root, for an escaped group; = record, for an
//            overflow group),
// which equals sum_c w~[r][c] x[b][c] with w~ the original-basis weights
// (the doubled coordinates P = 2p account for the 1/2).
//
// Three launches:
//  k_gv_prep  (a) per activation row and 2048-column segment: xr in fp32
//             (group-major) and in fp16 scaled by a power of two chosen
//             from the row's largest |x| so that no value can overflow fp16,
//             stored in the order in which the MMA B fragments are read;
//             (b) per weight row: a dense byte map group -> root + 1 (0: no
//             escape) from the escape records, in any record order.
//  k_gv_main  tensor cores: mma.sync m16n8k16, A = codewords (16 weight rows
//             x 16 coordinates), B = activations (16 coordinates x 8 batch
//             rows), fp32 accumulate.  The work -- 256-row blocks times
//             256-column chunks times 8 k-steps -- is split into equal
//             contiguous k-step ranges, one per CTA (one resident CTA per
//             SM); the 16 warps of a CTA, one 16-row tile each, take
//             different rows of the same range, so they read the same
//             activation fragments (L1 hits).  The first
//             49,152 codeword words live in shared memory (a shared-memory
//             gather costs a few wavefronts per warp, a global one up to one
//             per lane); the rest are read through L1.  Indices and root-map
//             bytes of the next chunk are loaded while the current one is
//             multiplied.  Escape roots are added to the codeword bytes before
//             the fp16 conversion.  Partial sums go to a per-(row block, CTA)
//             slot of the workspace.
//  k_gv_fin   per weight row: the partial slots in a fixed order, the
//             overflow records (CUDA cores, fp32 activations; lanes split
//             over records and batch rows), the scale, bf16 output.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace e8q {

// Core codeword k as 8 nibbles: nibble i (bits 4i..4i+3) = P_i + 8.
__device__ __align__(16) uint32_t g_gv_tab[65536];

constexpr int kGvBlockRows = 256;  // rows per row block (one CTA's rows): 16-row MMA tiles over the warps
constexpr int kGvChunkCols = 256;  // columns per chunk: 32 groups, 8 k-steps
constexpr int kGvTabN = 49152;     // codeword words held in shared memory
constexpr int kGvMaxCtas = 160;    // upper bound on main-kernel CTAs (workspace sizing)
constexpr int kGvSegCols = 2048;   // activation columns per prep CTA
constexpr int kGvPassTiles = 8;    // batch tiles of 8 per main-kernel pass
constexpr size_t kGvTabBytes = size_t{kGvTabN} * 4;
constexpr size_t kGvRootBytes = 256 * 8;
constexpr size_t kGvSmemBytes = kGvTabBytes + kGvRootBytes;

struct GvGeom {
    int32_t rows, cols, gpr, batch;
    int32_t nbt;       // batch tiles of 8
    int32_t nchunks;   // 256-column chunks (last one may be partial)
    int32_t nrb;       // 256-row blocks
    int32_t nctas;     // main-kernel CTAs with work
    int32_t maxslots;  // partial slots per row block
    int32_t mstride;   // root-map bytes per row (32 * nchunks)
    int32_t seg_cols;  // prep segment
    int32_t nseg;
    int32_t logb;
    int64_t ksteps;    // nrb * nchunks * 8
};

inline GvGeom gv_geometry(int64_t rows, int64_t cols, int batch, int logb, int ctas) {
    GvGeom g;
    g.rows = static_cast<int32_t>(rows);
    g.cols = static_cast<int32_t>(cols);
    g.gpr = g.cols / 8;
    g.batch = batch;
    g.nbt = (batch + 7) / 8;
    g.nchunks = (g.cols + kGvChunkCols - 1) / kGvChunkCols;
    g.nrb = (g.rows + kGvBlockRows - 1) / kGvBlockRows;
    g.ksteps = static_cast<int64_t>(g.nrb) * g.nchunks * 8;
    g.nctas = static_cast<int32_t>(g.ksteps < ctas ? g.ksteps : ctas);
    if (g.nctas < 1) g.nctas = 1;
    // a row block's k-steps meet at most ceil(KS / per) + 1 CTA ranges
    const int64_t per = g.ksteps / g.nctas > 0 ? g.ksteps / g.nctas : 1;
    const int64_t ks = static_cast<int64_t>(g.nchunks) * 8;
    int64_t slots = (ks + per - 1) / per + 1;
    if (slots > g.nctas) slots = g.nctas;
    g.maxslots = static_cast<int32_t>(slots);
    g.mstride = 32 * g.nchunks;
    g.seg_cols = g.cols < kGvSegCols ? g.cols : kGvSegCols;
    g.nseg = g.seg_cols > 0 ? (g.cols + g.seg_cols - 1) / g.seg_cols : 0;
    g.logb = logb;
    return g;
}

struct GvWs {
    size_t x32, x16, xe, map, part, total;
};
inline size_t gv_round(size_t x) { return (x + 255) / 256 * 256; }
inline GvWs gv_workspace(const GvGeom& g) {
    GvWs w;
    w.x32 = 0;
    w.x16 = w.x32 + gv_round(static_cast<size_t>(g.batch) * g.cols * 4);
    w.xe = w.x16 + gv_round(static_cast<size_t>(g.nchunks) * g.nbt * 8 * 32 * 16);
    w.map = w.xe + gv_round(static_cast<size_t>(g.nbt) * 8 * 4);
    w.part = w.map + gv_round(static_cast<size_t>(g.rows) * g.mstride);
    const size_t slots = static_cast<size_t>(g.nrb) * g.maxslots * g.batch * kGvBlockRows * 4;
    w.total = w.part + gv_round(slots);
    return w;
}

// The CTA whose k-step range holds k-step u (ranges: [floor(wT/W), floor((w+1)T/W))).
__host__ __device__ __forceinline__ int64_t gv_cta_of(int64_t u, int64_t T, int64_t W) {
    return ((u + 1) * W - 1) / T;
}

// ---------------------------------------------------------------------------
// prep
// ---------------------------------------------------------------------------
struct GvPrepParams {
    const uint16_t* x;  // bf16 [batch][cols]
    const int8_t* signs;
    float* x32;         // [groups][batch][8]: one group's 8 values of every batch row together
    uint4* x16;         // [nchunks][nbt][8 k-steps][32 lanes] x 8 halves
    float* xe;          // [batch]: 2^e, x16 = xr * 2^-e
    const e8q_escape* esc;
    const int64_t* esc_rp;
    uint8_t* map;       // [rows][mstride]: root + 1 of an escaped group, else 0
    long long esc_n;
    long long group_base;
    GvGeom g;
    int32_t n_xcta;     // CTAs of part (a)
};

__device__ __forceinline__ long long gv_clamp(long long v, long long lo, long long hi) {
    return v < lo ? lo : (v > hi ? hi : v);
}

__device__ __forceinline__ unsigned pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const unsigned*>(&h);
}

// Exponent e of one activation row (a CTA of 256 threads): |xr_i| <=
// sqrt(B) max|x|, so xr * 2^-e stays below 2^15 and cannot overflow fp16.
// s_red: 8 words of shared memory.
__device__ inline int gv_row_exponent(const uint16_t* xb, int C, int logb, unsigned* s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // largest |x| of the row, as bf16 magnitude bits (integer order = value order)
    unsigned m = 0;
    for (int i0 = 0; i0 < C / 8; i0 += 8 * 256) {
        uint4 v[8];  // all loads of a round before their use
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + threadIdx.x + 256 * k;
            v[k] = i < C / 8 ? __ldg(reinterpret_cast<const uint4*>(xb) + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const unsigned w4[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) m = max(m, max(w4[e] & 0x7FFFu, (w4[e] >> 16) & 0x7FFFu));
        }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = s_red[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) m = max(m, s_red[k]);
    int e = 0;
    if (m != 0 && m < 0x7F80u) {
        const float bound = __uint_as_float(m << 16) * sqrtf(static_cast<float>(1 << logb)) * 1.0001f;
        int k;
        frexpf(bound, &k);
        e = k - 15;
        e = e < -126 ? -126 : (e > 126 ? 126 : e);
    }
    return e;
}

// buf[0 .. n) = H_B (d (.) x)[c0 .. c0 + n) without the 1/sqrt(B) (a CTA of
// 256 threads; n a multiple of B).
__device__ inline void gv_rotate_segment(float* buf, const uint16_t* xb, const int8_t* signs, int c0, int n, int logb) {
    for (int i = threadIdx.x; i < n; i += 256) {
        const float v = __uint_as_float(static_cast<unsigned>(xb[c0 + i]) << 16);
        buf[i] = signs[c0 + i] < 0 ? -v : v;
    }
    __syncthreads();
    if (logb > 0) fwht_smem(buf, n, logb);
}

__global__ void __launch_bounds__(256) k_gv_prep(const __grid_constant__ GvPrepParams p) {
    __shared__ __align__(16) float buf[kGvSegCols];
    __shared__ unsigned s_red[8];
    pdl_launch_dependents();
    const GvGeom& G = p.g;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (static_cast<int>(blockIdx.x) < p.n_xcta) {
        const int b = blockIdx.x / G.nseg, seg = blockIdx.x % G.nseg;
        const int C = G.cols;
        const uint16_t* xb = p.x + static_cast<size_t>(b) * C;
        const int e = gv_row_exponent(xb, C, G.logb, s_red);
        const float down = __uint_as_float(static_cast<unsigned>(127 - e) << 23);  // 2^-e
        const int c0 = seg * G.seg_cols;
        const int n = min(G.seg_cols, C - c0);
        gv_rotate_segment(buf, xb, p.signs, c0, n, G.logb);
        const float inv = 1.0f / sqrtf(static_cast<float>(1 << G.logb));
        for (int t = threadIdx.x; t < n / 8; t += 256) {
            const int col = c0 + 8 * t;
            float4* xg = reinterpret_cast<float4*>(p.x32 + (static_cast<size_t>(col >> 3) * G.batch + b) * 8);
            xg[0] = make_float4(buf[8 * t] * inv, buf[8 * t + 1] * inv, buf[8 * t + 2] * inv, buf[8 * t + 3] * inv);
            xg[1] = make_float4(buf[8 * t + 4] * inv, buf[8 * t + 5] * inv, buf[8 * t + 6] * inv, buf[8 * t + 7] * inv);
            const int c = col >> 8, gc = (col & 255) >> 3, q = gc >> 3, j = gc & 7;
            const int L = 4 * (b & 7) + q;
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = buf[8 * t + i] * inv * down;
            uint4 o;
            o.x = pack_half2(v[0], v[1]);
            o.y = pack_half2(v[2], v[3]);
            o.z = pack_half2(v[4], v[5]);
            o.w = pack_half2(v[6], v[7]);
            p.x16[((static_cast<size_t>(c) * G.nbt + (b >> 3)) * 8 + j) * 32 + L] = o;
        }
        if (seg == 0 && threadIdx.x == 0) p.xe[b] = __uint_as_float(static_cast<unsigned>(127 + e) << 23);
        return;
    }
    // (b) root map of one weight row per warp: clear, then scatter the row's records
    if (!p.esc_rp) return;
    const int r = (blockIdx.x - p.n_xcta) * 8 + warp;
    if (r >= G.rows) return;
    uint8_t* mrow = p.map + static_cast<size_t>(r) * G.mstride;
    for (int i = lane; i < G.mstride / 16; i += 32) reinterpret_cast<uint4*>(mrow)[i] = make_uint4(0, 0, 0, 0);
    __syncwarp();
    const long long e0 = gv_clamp(p.esc_rp[r], 0, p.esc_n);
    const long long e1 = gv_clamp(p.esc_rp[r + 1], e0, p.esc_n);
    const long long g0 = p.group_base + static_cast<long long>(r) * G.gpr;
    // records in rounds of 8 per lane: all loads of a round before its stores
    for (long long k0 = e0; k0 < e1; k0 += 8 * 32) {
        uint2 rec[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const long long k = k0 + lane + 32 * i;
            rec[i] = k < e1 ? __ldcs(reinterpret_cast<const uint2*>(p.esc + k)) : make_uint2(0u, 0xFF0000u);  // root 255: none
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const long long gl = static_cast<long long>(rec[i].x) - g0;  // group
            const unsigned root = (rec[i].y >> 16) & 0xFFu;
            if (gl >= 0 && gl < G.gpr && root < 240) mrow[gl] = static_cast<uint8_t>(root + 1);
        }
    }
}

// ---------------------------------------------------------------------------
// main
// ---------------------------------------------------------------------------
struct GvMainParams {
    const uint16_t* idx;
    const uint4* x16;
    const uint8_t* map;  // null: no escapes
    float* part;         // [nrb][maxslots][256 rows][batch]
    GvGeom g;
    int32_t v0;          // first batch tile of this pass
    int32_t vec_idx;     // index rows 16-byte aligned (gpr % 8 == 0, aligned base)
};

__device__ __forceinline__ void mma_f16(float (&d)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3, unsigned b0,
                                        unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ unsigned hsub2_bits(unsigned a, unsigned b) {
    unsigned r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// 8 indices of one row: groups gs .. gs+7 (0 past the row end).
__device__ __forceinline__ uint4 gv_idx8(const uint16_t* rowp, int gs, int gpr, bool vec) {
    if (vec && gs + 8 <= gpr) return __ldcs(reinterpret_cast<const uint4*>(rowp + gs));
    unsigned h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = (gs + i < gpr) ? static_cast<unsigned>(rowp[gs + i]) : 0u;
    return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
}

// Rows of codeword slot r (0 .. 2RT-1) inside the warp: tile r>>1, +8 for odd r.
__device__ __forceinline__ int gv_row_in_warp(int r, int g) { return 16 * (r >> 1) + 8 * (r & 1) + g; }

template <int RT>
struct GvVisit {
    uint4 idx[2 * RT];  // 8 indices per codeword row
    uint2 map[2 * RT];  // 8 root-map bytes per codeword row
};

template <int RT>
__device__ __forceinline__ void gv_load_idx(const GvMainParams& p, int rb, int c, int warp, int g, int q,
                                            GvVisit<RT>& d) {
    const GvGeom& G = p.g;
    const int gs = 32 * c + 8 * q;
#pragma unroll
    for (int r = 0; r < 2 * RT; ++r) {
        const int row = rb * kGvBlockRows + warp * 16 * RT + gv_row_in_warp(r, g);
        d.idx[r] = row < G.rows ? gv_idx8(p.idx + static_cast<size_t>(row) * G.gpr, gs, G.gpr, p.vec_idx != 0)
                                : make_uint4(0, 0, 0, 0);
    }
}

template <int RT>
__device__ __forceinline__ void gv_load_map(const GvMainParams& p, int rb, int c, int warp, int g, int q,
                                            GvVisit<RT>& d) {
    const GvGeom& G = p.g;
    const int gs = 32 * c + 8 * q;
#pragma unroll
    for (int r = 0; r < 2 * RT; ++r) {
        const int row = rb * kGvBlockRows + warp * 16 * RT + gv_row_in_warp(r, g);
        d.map[r] = (row < G.rows && p.map)
                       ? __ldcg(reinterpret_cast<const uint2*>(p.map + static_cast<size_t>(row) * G.mstride + gs))
                       : make_uint2(0, 0);
    }
}

__device__ __forceinline__ unsigned gv_comp(const uint4& v, int k) {
    return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

// Codeword word of codeword row r at k-step j (shared table, else L1).
template <int RT>
__device__ __forceinline__ unsigned gv_word(const GvVisit<RT>& cv, const uint32_t* s_tab, int r, int j) {
    const unsigned comp = gv_comp(cv.idx[r], j >> 1);
    const unsigned id = (j & 1) ? (comp >> 16) : (comp & 0xFFFFu);
    return id < static_cast<unsigned>(kGvTabN) ? s_tab[id] : __ldg(g_gv_tab + id);
}

// Codeword pairs (P_2k, P_2k+1) in fp16 of the codeword rows at k-step j.
template <int RT, bool ESC>
__device__ __forceinline__ void gv_decode(const GvVisit<RT>& cv, const unsigned (&wd)[2 * RT], const uint2* s_root,
                                          int j, unsigned (&pr)[2 * RT][4]) {
#pragma unroll
    for (int r = 0; r < 2 * RT; ++r) {
        const unsigned w = wd[r];
        unsigned lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu, bias;
        if (ESC) {
            const unsigned root = ((j < 4 ? cv.map[r].x : cv.map[r].y) >> (8 * (j & 3))) & 0xFFu;
            const uint2 rb = s_root[root];
            lo += rb.x;
            hi += rb.y;
            bias = 0x640A640Au;  // 1034 = 1024 + 8 + 2
        } else {
            bias = 0x64086408u;  // 1032 = 1024 + 8
        }
        pr[r][0] = hsub2_bits(prmt(lo, hi, 0x8480u) | 0x64006400u, bias);
        pr[r][1] = hsub2_bits(prmt(lo, hi, 0x8581u) | 0x64006400u, bias);
        pr[r][2] = hsub2_bits(prmt(lo, hi, 0x8682u) | 0x64006400u, bias);
        pr[r][3] = hsub2_bits(prmt(lo, hi, 0x8783u) | 0x64006400u, bias);
    }
}

template <int RT, int NBP>
__device__ __forceinline__ void gv_mma(float (&acc)[RT][NBP][4], const unsigned (&pr)[2 * RT][4],
                                       const uint4 (&xb)[NBP]) {
#pragma unroll
    for (int u = 0; u < NBP; ++u)
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            mma_f16(acc[t][u], pr[2 * t][0], pr[2 * t + 1][0], pr[2 * t][1], pr[2 * t + 1][1], xb[u].x, xb[u].y);
            mma_f16(acc[t][u], pr[2 * t][2], pr[2 * t + 1][2], pr[2 * t][3], pr[2 * t + 1][3], xb[u].z, xb[u].w);
        }
}

// Activation fragments of k-step j for the pass's batch tiles (0 where the
// batch row or the group does not exist).
template <int NBP>
__device__ __forceinline__ void gv_load_x(const uint4* xs, const bool (&bok)[NBP], bool jok, int j, int lane,
                                          uint4 (&xb)[NBP]) {
#pragma unroll
    for (int u = 0; u < NBP; ++u)
        xb[u] = (bok[u] && jok) ? __ldg(xs + static_cast<size_t>(u) * 256 + j * 32 + lane) : make_uint4(0, 0, 0, 0);
}

template <int RT, int NBP, bool ESC>
__device__ __forceinline__ void gv_visit(float (&acc)[RT][NBP][4], const GvVisit<RT>& cv, const uint32_t* s_tab,
                                         const uint2* s_root, const uint4* xs, const bool (&bok)[NBP], int lim, int j0,
                                         int j1, int lane) {
    if (RT * NBP <= 2) {
        // every codeword word and activation fragment of the chunk up front:
        // one exposed latency per chunk
        unsigned wd[8][2 * RT];
        uint4 xa[8][NBP];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int r = 0; r < 2 * RT; ++r) wd[j][r] = (j >= j0 && j < j1) ? gv_word<RT>(cv, s_tab, r, j) : 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) gv_load_x<NBP>(xs, bok, j < lim && j >= j0 && j < j1, j, lane, xa[j]);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j >= j0 && j < j1) {
                unsigned pr[2 * RT][4];
                gv_decode<RT, ESC>(cv, wd[j], s_root, j, pr);
                gv_mma<RT, NBP>(acc, pr, xa[j]);
            }
    } else if (NBP >= 8) {
        // no room for a second set of fragments: load at the k-step
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j >= j0 && j < j1) {
                uint4 xb[NBP];
                unsigned wd[2 * RT];
#pragma unroll
                for (int r = 0; r < 2 * RT; ++r) wd[r] = gv_word<RT>(cv, s_tab, r, j);
                gv_load_x<NBP>(xs, bok, j < lim, j, lane, xb);
                unsigned pr[2 * RT][4];
                gv_decode<RT, ESC>(cv, wd, s_root, j, pr);
                gv_mma<RT, NBP>(acc, pr, xb);
            }
    } else {
        uint4 xb[NBP], xn[NBP];
        unsigned wd[2 * RT], wn[2 * RT];
#pragma unroll
        for (int r = 0; r < 2 * RT; ++r) wd[r] = gv_word<RT>(cv, s_tab, r, j0);
        gv_load_x<NBP>(xs, bok, j0 < lim, j0, lane, xb);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j >= j0 && j < j1) {
                if (j + 1 < j1) {
                    gv_load_x<NBP>(xs, bok, j + 1 < lim, j + 1, lane, xn);
#pragma unroll
                    for (int r = 0; r < 2 * RT; ++r) wn[r] = gv_word<RT>(cv, s_tab, r, j + 1);
                }
                unsigned pr[2 * RT][4];
                gv_decode<RT, ESC>(cv, wd, s_root, j, pr);
                gv_mma<RT, NBP>(acc, pr, xb);
#pragma unroll
                for (int u = 0; u < NBP; ++u) xb[u] = xn[u];
#pragma unroll
                for (int r = 0; r < 2 * RT; ++r) wd[r] = wn[r];
            }
    }
}

template <int RT, int NBP>
__device__ __forceinline__ void gv_flush(const GvMainParams& p, float (&acc)[RT][NBP][4], int rb, int warp, int g,
                                         int q) {
    const GvGeom& G = p.g;
    const long long ks = static_cast<long long>(G.nchunks) * 8;
    const long long slot = static_cast<long long>(blockIdx.x) - gv_cta_of(static_cast<long long>(rb) * ks, G.ksteps, G.nctas);
    if (slot >= 0 && slot < G.maxslots) {
        float* base = p.part + ((static_cast<size_t>(rb) * G.maxslots + slot) * kGvBlockRows + warp * 16 * RT) *
                                   G.batch;
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int u = 0; u < NBP; ++u)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int b = 8 * (p.v0 + u) + 2 * q + (k & 1);
                    const int ri = 16 * t + g + 8 * (k >> 1);
                    if (b < G.batch) base[static_cast<size_t>(ri) * G.batch + b] = acc[t][u][k];
                }
    }
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int u = 0; u < NBP; ++u)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[t][u][k] = 0.f;
}

// Root byte vectors: entry 0 = no root, entry 1 + i = root i; bytes R + 2,
// even coordinates in .x, odd coordinates in .y.
__device__ __forceinline__ uint2 gv_root_entry(int i) {
    if (i == 0) return make_uint2(0x02020202u, 0x02020202u);
    if (i > 240) return make_uint2(0u, 0u);
    const uint2 rw = g_root8[i - 1];
    unsigned lo = 0, hi = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int c_even = static_cast<int8_t>(((k < 2 ? rw.x : rw.y) >> (16 * (k & 1))) & 0xFF);
        const int c_odd = static_cast<int8_t>(((k < 2 ? rw.x : rw.y) >> (16 * (k & 1) + 8)) & 0xFF);
        lo |= static_cast<unsigned>(c_even + 2) << (8 * k);
        hi |= static_cast<unsigned>(c_odd + 2) << (8 * k);
    }
    return make_uint2(lo, hi);
}

// RT 16-row tiles per warp, 16 / RT warps per CTA (256 rows); NBP batch tiles of 8.
template <int RT, int NBP>
__global__ void __launch_bounds__(512 / RT, 1) k_gv_main(const __grid_constant__ GvMainParams p) {
    constexpr int kThreads = 512 / RT;
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t* s_tab = reinterpret_cast<uint32_t*>(smem);
    uint2* s_root = reinterpret_cast<uint2*>(smem + kGvTabBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const GvGeom& G = p.g;
    const long long cta = blockIdx.x;
    const long long lo = cta * G.ksteps / G.nctas, hi = (cta + 1) * G.ksteps / G.nctas;
    const long long vbeg = lo >> 3, vend = (hi + 7) >> 3;
    int rb = static_cast<int>(vbeg / G.nchunks), c = static_cast<int>(vbeg % G.nchunks);
    pdl_launch_dependents();
    // prologue independent of the prep kernel: first indices, shared tables
    GvVisit<RT> cur;
    if (lo < hi) gv_load_idx<RT>(p, rb, c, warp, g, q, cur);
    for (int i = threadIdx.x; i < kGvTabN / 4; i += kThreads)
        reinterpret_cast<uint4*>(s_tab)[i] = __ldg(reinterpret_cast<const uint4*>(g_gv_tab) + i);
    for (int i = threadIdx.x; i < 256; i += kThreads) s_root[i] = gv_root_entry(i);
    __syncthreads();
    pdl_wait();  // activations and root map written by the prep kernel
    if (lo >= hi) return;
    gv_load_map<RT>(p, rb, c, warp, g, q, cur);

    bool bok[NBP];
#pragma unroll
    for (int u = 0; u < NBP; ++u) bok[u] = 8 * (p.v0 + u) + g < G.batch;

    float acc[RT][NBP][4];
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int u = 0; u < NBP; ++u)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[t][u][k] = 0.f;

    int cur_rb = rb;
    for (long long v = vbeg; v < vend; ++v) {
        GvVisit<RT> nxt;
        int nrb = rb, nc = c + 1;
        if (nc == G.nchunks) {
            nc = 0;
            ++nrb;
        }
        if (v + 1 < vend) {
            gv_load_idx<RT>(p, nrb, nc, warp, g, q, nxt);
            gv_load_map<RT>(p, nrb, nc, warp, g, q, nxt);
        }
        if (rb != cur_rb) {
            gv_flush<RT, NBP>(p, acc, cur_rb, warp, g, q);
            cur_rb = rb;
        }
        const int j0 = v == vbeg ? static_cast<int>(lo & 7) : 0;
        const int j1 = v == vend - 1 ? static_cast<int>(((hi - 1) & 7) + 1) : 8;
        const int vg = G.gpr - 32 * c < 32 ? G.gpr - 32 * c : 32;  // valid groups in this chunk
        const int lim = vg - 8 * q;
        const uint4* xs = p.x16 + (static_cast<size_t>(c) * G.nbt + p.v0) * 256;
        unsigned any = 0;
#pragma unroll
        for (int r = 0; r < 2 * RT; ++r) any |= cur.map[r].x | cur.map[r].y;
        if (__any_sync(0xFFFFFFFFu, any != 0))
            gv_visit<RT, NBP, true>(acc, cur, s_tab, s_root, xs, bok, lim, j0, j1, lane);
        else
            gv_visit<RT, NBP, false>(acc, cur, s_tab, s_root, xs, bok, lim, j0, j1, lane);
        cur = nxt;
        rb = nrb;
        c = nc;
    }
    gv_flush<RT, NBP>(p, acc, cur_rb, warp, g, q);
}

// ---------------------------------------------------------------------------
// finalize
// ---------------------------------------------------------------------------
struct GvFinParams {
    const float* part;
    const float* xe;
    const float* x32;
    const float* scale;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    uint16_t* y;  // bf16 [batch][rows]
    long long ovf_n;
    long long group_base;
    GvGeom g;
    int32_t bl_log;  // log2 of the batch lanes: lanes = record lane * BL + batch lane
};

// Lanes = record lane rl (slots / overflow records) x batch lane bl; each
// lane holds KB batch rows bl, bl + BL, ...; one shuffle reduction over rl.
template <int KB>
__global__ void __launch_bounds__(256) k_gv_fin(const __grid_constant__ GvFinParams p) {
    pdl_wait();  // partial sums of the main kernel
    const GvGeom& G = p.g;
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= G.rows) return;
    const int BL = 1 << p.bl_log, RL = 32 >> p.bl_log;
    const int bl = lane & (BL - 1), rl = lane >> p.bl_log;
    const int rb = r / kGvBlockRows, ri = r % kGvBlockRows;
    const long long ks = static_cast<long long>(G.nchunks) * 8;
    const long long c0 = gv_cta_of(static_cast<long long>(rb) * ks, G.ksteps, G.nctas);
    const long long c1 = gv_cta_of(static_cast<long long>(rb) * ks + ks - 1, G.ksteps, G.nctas);
    const int nsl = static_cast<int>(c1 - c0 + 1 < G.maxslots ? c1 - c0 + 1 : G.maxslots);
    const float* pb = p.part + (static_cast<size_t>(rb) * G.maxslots * kGvBlockRows + ri) * G.batch;
    const size_t sstride = static_cast<size_t>(kGvBlockRows) * G.batch;
    float acc[KB];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
        const int b = bl + BL * k;
        float v = 0.f;
        if (b < G.batch) {
#pragma unroll 4
            for (int sl = rl; sl < nsl; sl += RL) v += __ldcg(pb + sl * sstride + b);
            v *= p.xe[b];
        }
        acc[k] = v;
    }
    if (p.ovf_rp) {
        const long long o0 = gv_clamp(p.ovf_rp[r], 0, p.ovf_n);
        const long long o1 = gv_clamp(p.ovf_rp[r + 1], o0, p.ovf_n);
        const long long g0 = p.group_base + static_cast<long long>(r) * G.gpr;
        for (long long oc = o0; oc < o1; oc += 4 * RL) {
            // up to 4 records per lane: records first, then activations
            int gls[4];
            int cw[4][4];  // coordinate pairs as packed int16
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const long long o = oc + rl + static_cast<long long>(RL) * i;
                gls[i] = -1;
                if (o < o1) {
                    const unsigned* rp = reinterpret_cast<const unsigned*>(p.ovf + o);
                    const long long gl = static_cast<long long>(__ldg(rp)) - g0;
                    if (gl >= 0 && gl < G.gpr) gls[i] = static_cast<int>(gl);
#pragma unroll
                    for (int k = 0; k < 4; ++k) cw[i][k] = static_cast<int>(__ldg(rp + 1 + k));
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (gls[i] < 0) continue;
                // the record's coordinates as exact floats, once: an int16 x added to
                // the bits of 1.5 * 2^23 is that float plus x
                float pc[8];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int lo = static_cast<int>(static_cast<int16_t>(cw[i][c] & 0xFFFF)), hi = cw[i][c] >> 16;
                    pc[2 * c] = __int_as_float(0x4B400000 + lo) - 12582912.f;
                    pc[2 * c + 1] = __int_as_float(0x4B400000 + hi) - 12582912.f;
                }
                const float4* xc = reinterpret_cast<const float4*>(p.x32 + static_cast<size_t>(gls[i]) * G.batch * 8);
#pragma unroll
                for (int k = 0; k < KB; ++k) {
                    const int b = bl + BL * k;
                    if (b < G.batch) {
                        const float4 u = __ldg(xc + 2 * b), t = __ldg(xc + 2 * b + 1);
                        float a = acc[k];
                        a = fmaf(pc[0], u.x, a);
                        a = fmaf(pc[1], u.y, a);
                        a = fmaf(pc[2], u.z, a);
                        a = fmaf(pc[3], u.w, a);
                        a = fmaf(pc[4], t.x, a);
                        a = fmaf(pc[5], t.y, a);
                        a = fmaf(pc[6], t.z, a);
                        a = fmaf(pc[7], t.w, a);
                        acc[k] = a;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < KB; ++k)
        for (int off = BL; off < 32; off <<= 1) acc[k] += __shfl_xor_sync(0xFFFFFFFFu, acc[k], off);
    if (rl == 0) {
        const float s = 0.5f * p.scale[r];
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            const int b = bl + BL * k;
            if (b < G.batch)
                p.y[static_cast<size_t>(b) * G.rows + r] = __bfloat16_as_ushort(__float2bfloat16_rn(s * acc[k]));
        }
    }
}

}  // namespace e8q
