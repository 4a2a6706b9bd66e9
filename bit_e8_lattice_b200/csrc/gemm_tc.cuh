// K5 for a batch of activation rows (prefill and the QAT forward, batch 64
// and up) on the 5th-generation tensor cores ("E8-QAT", abstract: decoding
// throughput of the 2-bit representation):
//
//   y[t][r] = s_r / 2 * sum_g < P_rg , xr_t[8g .. 8g+7] >,
//   xr_t    = H_B (d (.) x_t) / sqrt(B)            (blockwise),
//   P_rg    = core[idx_rg] (+ root, escaped group; = record, overflow group),
//
// without materialising the dequantised weights: the codewords go from the
// 16-bit indices straight into the tensor cores' shared-memory operand.
//
// Launches:
//  k_gm_prep  (a) per token row (the whole row in shared memory, one pass
//             of the blockwise transform): xr * 2^-e in fp16, e chosen from
//             the row's largest |x| (no fp16 overflow), stored as an
//             operand image: per (256-token
//             tile, 32-column K tile) one contiguous 16 KB block in the
//             K-major, no-swizzle core-matrix layout, so that one 1-D bulk
//             copy stages it;
//             (b) per weight row: a 16-bit map group -> root + 1 (escape),
//             0x8000 | the record's place among the row's overflow records,
//             or 0; and a flag for rows holding an overflow point with a
//             coordinate beyond fp16's exact integers (|P_i| > 2048).
//  k_gm_main  persistent CTAs over units (128-row tile, 256-token tile, K
//             split), one CTA per SM, 9 warps:
//             - 16 producer warps, four threads per weight row of the tile,
//               one group each per 32-column K tile: the thread turns the
//               group's index into its codeword (shared-memory copy of the
//               table's first 32,768 words, the rest through L1), adds the
//               escape root or substitutes the overflow record, and writes
//               the group as fp16 into the A stage; indices, map entries and
//               row record offsets are loaded six K tiles ahead, table words
//               and records three ahead.  One elected arrival per warp on a
//               4-stage ring of mbarriers;
//             - 1 copy warp: one thread starts the bulk copy of each K
//               tile's activation image into the B stage as soon as the
//               stage is free (up to four K tiles ahead);
//             - 1 MMA warp: one thread issues two M = 128, N = tokens,
//               K = 16 kind::f16 MMAs per stage into one of two tensor-memory
//               accumulators (256 columns each) and commits the stage back;
//             - 4 epilogue warps read a finished accumulator (tcgen05.ld),
//               and write bf16 y (one split) or fp32 partial sums (several),
//               overlapping the next unit's MMAs.
//  k_gm_fin   (several K splits only) per output: the splits' partial sums
//             in a fixed order, the scale, bf16.
// Overflow points with a coordinate beyond +-2048 are left out of the
// operand and added on CUDA cores from the same fp16 activations.
// Every wait is bounded; one that gives up sets the call's error word.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemv.cuh"
#include "ptx.cuh"

namespace e8q {

constexpr int kGmRows = 128;     // M: weight rows per tile (tensor-memory lanes)
constexpr int kGmKCols = 32;     // K columns per stage: 4 groups, two MMAs of K = 16
constexpr int kGmTok = 256;      // N: tokens per tile (one accumulator)
constexpr int kGmStages = 4;
constexpr int kGmProdWarps = 16;  // four threads per weight row
constexpr int kGmMmaWarp = kGmProdWarps;
constexpr int kGmCopyWarp = kGmProdWarps + 1;
constexpr int kGmThreads = (kGmProdWarps + 2 + 4) * 32;
constexpr int kGmWaitLimit = 1 << 20;
constexpr int kGmMaxSplit = 32;
constexpr int kGmPlanSms = 148;   // SM count the K-split plan is made for (results do not depend on the device)
constexpr int kGmMaxBatch = 65536;
constexpr int kGmTab = 32768;     // codeword words held in shared memory
constexpr int kGmFarP = 2048;     // fp16 holds every integer up to 2048 exactly
constexpr uint32_t kGmABytes = kGmRows * kGmKCols * 2;   // 8 KB
constexpr uint32_t kGmBBytes = kGmTok * kGmKCols * 2;    // 16 KB
constexpr uint32_t kGmStageBytes = kGmABytes + kGmBBytes;
constexpr size_t kGmSmemBytes = size_t{kGmStages} * kGmStageBytes + 256 * 8 + size_t{kGmTab} * 4;
static_assert(kGmSmemBytes <= 227 * 1024 - 256, "shared memory of one CTA");

struct GmGeom {
    int32_t rows, cols, gpr, batch;
    int32_t nrt;      // 128-row tiles
    int32_t nkt;      // 32-column K tiles
    int32_t ntt;      // 256-token tiles
    int32_t nsplit;   // K splits
    int32_t nunits;   // nrt * nsplit * ntt
    int32_t mstride;  // map entries per row (>= 4 nkt, a multiple of 8)
    int32_t seg_cols, nseg, logb;
};

// First K tile of split s.
__host__ __device__ __forceinline__ int gm_k0(const GmGeom& g, int s) {
    return static_cast<int>(static_cast<long long>(s) * g.nkt / g.nsplit);
}

// The K split: the split count with the least estimated time, each unit
// costing its K tiles times a per-stage time (tensor-core time for the
// token tile, at least the decode time), CTAs in rounds of kGmPlanSms, and
// several splits adding their fp32 partial sums' HBM traffic.
inline int gm_plan_split(int nrt, int nkt, int ntt, int batch, int rows) {
    const double tok = batch < kGmTok ? batch : kGmTok;
    const double stage_ns = tok * 0.75 > 150.0 ? tok * 0.75 : 150.0;
    const long long u0 = static_cast<long long>(nrt) * ntt;
    int best = 1;
    double best_t = 0.0;
    const int smax = nkt / 8 < kGmMaxSplit ? (nkt / 8 > 1 ? nkt / 8 : 1) : kGmMaxSplit;
    for (int s = 1; s <= smax; ++s) {
        const long long units = u0 * s;
        const long long rounds = (units + kGmPlanSms - 1) / kGmPlanSms;
        const double t = static_cast<double>(rounds) * ((nkt + s - 1) / s) * stage_ns +
                         (s > 1 ? static_cast<double>(s) * batch * rows * 8.0 / 6500.0 : 0.0);  // bytes at 6.5 TB/s, in ns
        if (s == 1 || t < best_t * 0.98) {
            best = s;
            best_t = t;
        }
    }
    return best;
}

inline GmGeom gm_geometry(int64_t rows, int64_t cols, int batch, int logb) {
    GmGeom g;
    g.rows = static_cast<int32_t>(rows);
    g.cols = static_cast<int32_t>(cols);
    g.gpr = g.cols / 8;
    g.batch = batch;
    g.nrt = (g.rows + kGmRows - 1) / kGmRows;
    g.nkt = (g.cols + kGmKCols - 1) / kGmKCols;
    g.ntt = (batch + kGmTok - 1) / kGmTok;
    g.nsplit = gm_plan_split(g.nrt, g.nkt, g.ntt, batch, g.rows);
    const long long units = static_cast<long long>(g.nrt) * g.nsplit * g.ntt;
    g.nunits = units > 0x7FFFFFFFll ? -1 : static_cast<int32_t>(units);
    g.mstride = (4 * g.nkt + 7) / 8 * 8;
    g.seg_cols = g.cols < kGvSegCols ? g.cols : kGvSegCols;
    g.nseg = g.seg_cols > 0 ? (g.cols + g.seg_cols - 1) / g.seg_cols : 0;
    g.logb = logb;
    return g;
}

struct GmWs {
    size_t err, img, xe, map, farf, part, total;
};
inline GmWs gm_workspace(const GmGeom& g) {
    GmWs w;
    w.err = 0;
    w.img = 256;
    w.xe = w.img + gv_round(static_cast<size_t>(g.ntt) * g.nkt * kGmBBytes);
    w.map = w.xe + gv_round(static_cast<size_t>(g.ntt) * kGmTok * 4);
    w.farf = w.map + gv_round(static_cast<size_t>(g.rows) * g.mstride * 2);
    w.part = w.farf + gv_round(static_cast<size_t>(g.rows));
    w.total = w.part + (g.nsplit > 1 ? gv_round(static_cast<size_t>(g.nsplit) * g.batch * g.rows * 4) : 0);
    return w;
}

// Byte offset of (row or token r, 8-column chunk kc) in a stage operand:
// core matrices of 8 rows x 16 bytes, the 4 chunks of a row group 128 bytes
// apart, row groups 512 bytes apart.
__host__ __device__ __forceinline__ uint32_t gm_core_off(int r, int kc) {
    return static_cast<uint32_t>(((r >> 3) * 4 + kc) * 128 + (r & 7) * 16);
}

// Byte offset of token t's 8 activations of group g in the operand image.
__device__ __forceinline__ size_t gm_img_off(const GmGeom& G, int t, int g) {
    return (static_cast<size_t>(t >> 8) * G.nkt + (g >> 2)) * kGmBBytes + gm_core_off(t & 255, g & 3);
}

// Shared-memory matrix descriptor for that layout (K-major, no swizzle):
// start >> 4, leading byte offset (next core matrix along K) 128 >> 4,
// stride byte offset (next 8 rows) 512 >> 4, descriptor version 1.
__device__ __forceinline__ uint64_t gm_sdesc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 16) |
           (static_cast<uint64_t>(512 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: fp32 D, fp16 A and B, both K-major, N, M = 128.
__device__ __forceinline__ uint32_t gm_idesc(int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kGmRows >> 4) << 24);
}

__device__ __forceinline__ void gm_wait(uint64_t* bar, unsigned parity, bool& dead) {
    if (dead) return;  // after one wait gave up, none blocks again: the kernel runs to its end
    for (int i = 0; i < kGmWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return;
    dead = true;
}

// Overflow record k as (group, 8 doubled coordinates).
__device__ __forceinline__ void gm_load_rec(const e8q_overflow* ovf, long long k, uint32_t& grp, uint4& c) {
    const uint32_t* rp = reinterpret_cast<const uint32_t*>(ovf) + 5 * k;
    grp = __ldg(rp);
    c = make_uint4(__ldg(rp + 1), __ldg(rp + 2), __ldg(rp + 3), __ldg(rp + 4));
}

// |coordinate| > 2048 for any of the 8 int16 coordinates.
__device__ __forceinline__ bool gm_far(const uint4& c) {
    const unsigned w[4] = {c.x, c.y, c.z, c.w};
    bool far = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int lo = static_cast<int16_t>(w[i] & 0xFFFFu), hi = static_cast<int16_t>(w[i] >> 16);
        far |= lo > kGmFarP || lo < -kGmFarP || hi > kGmFarP || hi < -kGmFarP;
    }
    return far;
}

// fp16 pairs of 8 integer coordinates (exact: |P_i| <= 2048).
__device__ __forceinline__ uint4 gm_coords_f16(const uint4& c) {
    const unsigned w[4] = {c.x, c.y, c.z, c.w};
    unsigned o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = pack_half2(static_cast<float>(static_cast<int16_t>(w[i] & 0xFFFFu)),
                          static_cast<float>(static_cast<int16_t>(w[i] >> 16)));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// ---------------------------------------------------------------------------
// prep
// ---------------------------------------------------------------------------
struct GmPrepParams {
    const uint16_t* x;  // bf16 [batch][cols]
    const int8_t* signs;
    unsigned char* img;  // [ntt][nkt] x 16 KB
    float* xe;           // [ntt * 256]: 2^e
    const e8q_escape* esc;
    const int64_t* esc_rp;
    long long esc_n;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    long long ovf_n;
    uint16_t* map;  // [rows][mstride]
    uint8_t* farf;  // [rows]
    unsigned long long* err;
    long long group_base;
    GmGeom g;
    int32_t n_xcta;  // CTAs of part (a): tokens rounded up to 16
};

__global__ void __launch_bounds__(256) k_gm_prep(const __grid_constant__ GmPrepParams p) {
    extern __shared__ __align__(16) float xs[];  // one token row (cols floats)
    __shared__ unsigned s_red[8];
    pdl_launch_dependents();
    const GmGeom& G = p.g;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.err = 0ull;
    if (static_cast<int>(blockIdx.x) < p.n_xcta) {
        const int t = blockIdx.x;
        const int gpad = 4 * G.nkt - G.gpr;  // zero groups past the row end
        if (t >= G.batch) {  // tokens up to the MMA's N: zeros
            for (int i = threadIdx.x; i < 4 * G.nkt; i += 256)
                *reinterpret_cast<uint4*>(p.img + gm_img_off(G, t, i)) = make_uint4(0, 0, 0, 0);
            return;
        }
        // the row, sign-flipped, into shared memory, and its largest |x| as
        // bf16 magnitude bits (integer order = value order)
        const uint4* xb = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * G.cols);
        unsigned m = 0;
        for (int i = threadIdx.x; i < G.gpr; i += 256) {
            const uint4 v = __ldg(xb + i);
            const unsigned w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const unsigned h = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                m = max(m, h & 0x7FFFu);
                const float f = __uint_as_float(h << 16);
                xs[8 * i + e] = __ldg(p.signs + 8 * i + e) < 0 ? -f : f;
            }
        }
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (lane == 0) s_red[warp] = m;
        __syncthreads();
        m = s_red[0];
#pragma unroll
        for (int k = 1; k < 8; ++k) m = max(m, s_red[k]);
        // |xr_i| <= sqrt(B) max|x|: pick e with sqrt(B) max|x| 2^-e < 2^15
        int e = 0;
        if (m != 0 && m < 0x7F80u) {
            const float bound = __uint_as_float(m << 16) * sqrtf(static_cast<float>(1 << G.logb)) * 1.0001f;
            int k;
            frexpf(bound, &k);
            e = k - 15;
            e = e < -126 ? -126 : (e > 126 ? 126 : e);
        }
        if (G.logb > 0) fwht_smem(xs, G.cols, G.logb);  // every block of the row at once
        const float f = __uint_as_float(static_cast<unsigned>(127 - e) << 23) / sqrtf(static_cast<float>(1 << G.logb));
        for (int i = threadIdx.x; i < G.gpr + gpad; i += 256) {
            uint4 o = make_uint4(0, 0, 0, 0);
            if (i < G.gpr) {
                const float* v = xs + 8 * i;
                o = make_uint4(pack_half2(v[0] * f, v[1] * f), pack_half2(v[2] * f, v[3] * f),
                               pack_half2(v[4] * f, v[5] * f), pack_half2(v[6] * f, v[7] * f));
            }
            *reinterpret_cast<uint4*>(p.img + gm_img_off(G, t, i)) = o;
        }
        if (threadIdx.x == 0) p.xe[t] = __uint_as_float(static_cast<unsigned>(127 + e) << 23);
        return;
    }
    // (b) one weight row per warp
    const int r = (blockIdx.x - p.n_xcta) * 8 + warp;
    if (r >= G.rows) return;
    uint16_t* mrow = p.map + static_cast<size_t>(r) * G.mstride;
    for (int i = lane; i < G.mstride / 8; i += 32) reinterpret_cast<uint4*>(mrow)[i] = make_uint4(0, 0, 0, 0);
    __syncwarp();
    const long long g0 = p.group_base + static_cast<long long>(r) * G.gpr;
    if (p.esc_rp) {
        const long long e0 = gv_clamp(p.esc_rp[r], 0, p.esc_n);
        const long long e1 = gv_clamp(p.esc_rp[r + 1], e0, p.esc_n);
        // records in rounds of 8 per lane: all loads of a round before its stores
        for (long long k0 = e0; k0 < e1; k0 += 8 * 32) {
            uint2 rec[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const long long k = k0 + lane + 32 * i;
                rec[i] = k < e1 ? __ldcs(reinterpret_cast<const uint2*>(p.esc + k)) : make_uint2(0u, 0xFF0000u);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const long long gl = static_cast<long long>(rec[i].x) - g0;
                const unsigned root = (rec[i].y >> 16) & 0xFFu;  // 255: no record
                if (gl >= 0 && gl < G.gpr && root < 240) mrow[gl] = static_cast<uint16_t>(root + 1);
            }
        }
    }
    bool far = false;
    if (p.ovf_rp) {
        const long long o0 = gv_clamp(p.ovf_rp[r], 0, p.ovf_n);
        const long long o1 = gv_clamp(p.ovf_rp[r + 1], o0, p.ovf_n);
        __syncwarp();  // escape entries first: a group listed twice ends as an overflow
        const long long o1c = o1 - o0 < 0x8000 ? o1 : o0 + 0x8000;  // offsets fit 15 bits
        for (long long k0 = o0; k0 < o1c; k0 += 4 * 32) {
            uint32_t grp[4];
            uint4 c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const long long k = k0 + lane + 32 * i;
                grp[i] = 0xFFFFFFFFu;
                c[i] = make_uint4(0, 0, 0, 0);
                if (k < o1c) gm_load_rec(p.ovf, k, grp[i], c[i]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const long long k = k0 + lane + 32 * i;
                const long long gl = static_cast<long long>(grp[i]) - g0;
                if (k < o1c && gl >= 0 && gl < G.gpr) {
                    mrow[gl] = static_cast<uint16_t>(0x8000u | static_cast<unsigned>(k - o0));
                    far |= gm_far(c[i]);
                }
            }
        }
    }
    far = __any_sync(0xFFFFFFFFu, far);
    if (lane == 0) p.farf[r] = far ? 1 : 0;
}

// ---------------------------------------------------------------------------
// main
// ---------------------------------------------------------------------------
struct GmMainParams {
    const uint16_t* idx;
    const uint16_t* map;
    const unsigned char* img;
    const float* xe;
    const float* scale;
    const uint8_t* farf;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    long long ovf_n;
    float* part;  // [nsplit][batch][rows] (several splits)
    uint16_t* y;  // bf16 [batch][rows]
    unsigned long long* err;
    long long group_base;
    GmGeom g;
};

struct GmUnit {
    int rt, tt, split, k0, k1;
};
__device__ __forceinline__ GmUnit gm_unit(const GmGeom& G, int u) {
    GmUnit U;
    U.rt = u % G.nrt;
    const int rest = u / G.nrt;
    U.split = rest % G.nsplit;
    U.tt = rest / G.nsplit;
    U.k0 = gm_k0(G, U.split);
    U.k1 = gm_k0(G, U.split + 1);
    return U;
}

// Sum over row r's overflow records with a coordinate beyond +-2048 of
// < P, x16_t > (the operand image's fp16 activations), in record order.
__device__ float gm_far_sum(const GmGeom& G, const unsigned char* img, const e8q_overflow* ovf,
                            const int64_t* ovf_rp, long long ovf_n, long long group_base, int r, int t) {
    const long long o0 = gv_clamp(ovf_rp[r], 0, ovf_n), o1 = gv_clamp(ovf_rp[r + 1], o0, ovf_n);
    const long long g0 = group_base + static_cast<long long>(r) * G.gpr;
    float acc = 0.f;
    for (long long k = o0; k < o1; ++k) {
        uint32_t grp;
        uint4 c;
        gm_load_rec(ovf, k, grp, c);
        const long long gl = static_cast<long long>(grp) - g0;
        if (gl < 0 || gl >= G.gpr || !gm_far(c)) continue;
        const uint4 xv = __ldcg(reinterpret_cast<const uint4*>(img + gm_img_off(G, t, static_cast<int>(gl))));
        const unsigned xw[4] = {xv.x, xv.y, xv.z, xv.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&xw[i]));
            acc = fmaf(static_cast<float>(static_cast<int16_t>(cw[i] & 0xFFFFu)), xf.x, acc);
            acc = fmaf(static_cast<float>(static_cast<int16_t>(cw[i] >> 16)), xf.y, acc);
        }
    }
    return acc;
}

__device__ __forceinline__ uint16_t gm_bf16(float v) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t*>(&h);
}

__global__ void __launch_bounds__(kGmThreads, 1) k_gm_main(const __grid_constant__ GmMainParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ __align__(8) uint64_t s_full[kGmStages], s_empty[kGmStages], s_accf[2], s_acce[2], s_done;
    __shared__ uint32_t s_taddr;
    unsigned char* stages = smem;
    uint2* s_root = reinterpret_cast<uint2*>(smem + kGmStages * kGmStageBytes);
    uint32_t* s_tab = reinterpret_cast<uint32_t*>(smem + kGmStages * kGmStageBytes + 256 * 8);
    const GmGeom& G = p.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nunits = G.nunits;
    pdl_launch_dependents();

    // tables (independent of the prep kernel), barriers, tensor memory
    for (int i = tid; i < 256; i += kGmThreads) s_root[i] = gv_root_entry(i);
    for (int i = tid; i < kGmTab / 4; i += kGmThreads)
        reinterpret_cast<uint4*>(s_tab)[i] = __ldg(reinterpret_cast<const uint4*>(g_gv_tab) + i);
    if (tid == 0) {
        for (int s = 0; s < kGmStages; ++s) {
            mbar_init(&s_full[s], kGmProdWarps + 1);  // one arrival per producer warp + the copy's expect_tx
            mbar_init(&s_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&s_accf[a], 1);
            mbar_init(&s_acce[a], 128);
        }
        mbar_init(&s_done, 1);
        fence_mbar_init();
    }
    if (warp == kGmMmaWarp) tmem_alloc(&s_taddr, 2 * kGmTok);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = s_taddr;
    pdl_wait();  // image, map and flags written by the prep kernel

    bool dead = false;
    if (warp < kGmProdWarps) {
        // ------------------------------------------------------ producers
        // Thread: weight row rl = 8 warp + (lane & 7) of the tile, group j =
        // lane >> 3 of every K tile.  At step q it decodes position q,
        // thread 0 starts the activation copy of position q + 2, it looks up
        // position q + 3 (table word or overflow record) and loads the
        // index, map entry and row record offset of position q + 6.
        const int rl = 8 * warp + (lane & 7), j = lane >> 3;
        struct Pos {
            int u, kt;
            GmUnit U;
        };
        auto first = [&]() {
            Pos x;
            x.u = blockIdx.x;
            x.U = gm_unit(G, x.u < nunits ? x.u : 0);
            x.kt = x.U.k0;
            return x;
        };
        auto next = [&](const Pos& x) {
            Pos y = x;
            if (++y.kt >= x.U.k1) {
                y.u = x.u + static_cast<int>(gridDim.x);
                y.U = gm_unit(G, y.u < nunits ? y.u : 0);
                y.kt = y.U.k0;
            }
            return y;
        };
        // index, map entry and row record offset of this thread's group of position x
        auto prefetch = [&](const Pos& x, unsigned& iv, unsigned& mv, long long& rb) {
            iv = 0u;
            mv = 0u;
            rb = 0;
            const int row = x.U.rt * kGmRows + rl, g = 4 * x.kt + j;
            if (x.u >= nunits || row >= G.rows || g >= G.gpr) return;
            iv = __ldg(p.idx + static_cast<size_t>(row) * G.gpr + g);
            mv = __ldcg(p.map + static_cast<size_t>(row) * G.mstride + g);
            if (p.ovf_rp) rb = __ldg(p.ovf_rp + row);
        };
        // the codeword word (table) or the overflow record's coordinates
        auto lookup = [&](unsigned iv, unsigned mv, long long rb, unsigned& w, uint4& c) {
            w = 0u;
            c = make_uint4(0, 0, 0, 0);
            if (mv & 0x8000u) {
                const long long k = gv_clamp(rb, 0, p.ovf_n) + (mv & 0x7FFFu);
                if (k < p.ovf_n) {
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.ovf) + 5 * k + 1;
                    c = make_uint4(__ldg(src), __ldg(src + 1), __ldg(src + 2), __ldg(src + 3));
                }
            } else {
                w = iv < static_cast<unsigned>(kGmTab) ? s_tab[iv] : __ldg(g_gv_tab + iv);
            }
        };
        // rings of 4 slots (position % 4): loaded values (index, map entry,
        // record offset), and looked-up values (word, map entry, coordinates)
        unsigned IV[4], MV[4], W[4], MD[4];
        long long RB[4];
        uint4 RC[4];
        Pos pd = first();  // decoded at this step (q)
        Pos pl = pd;       // loaded (q + 6)
        // prologue: loads of positions 0..2, then, as steps -3..-1, the
        // lookups of 0..2 and the loads of 3..5
        prefetch(pl, IV[0], MV[0], RB[0]);
        pl = next(pl);
        prefetch(pl, IV[1], MV[1], RB[1]);
        pl = next(pl);
        prefetch(pl, IV[2], MV[2], RB[2]);
        pl = next(pl);
        lookup(IV[0], MV[0], RB[0], W[0], RC[0]);
        MD[0] = MV[0];
        prefetch(pl, IV[3], MV[3], RB[3]);
        pl = next(pl);
        lookup(IV[1], MV[1], RB[1], W[1], RC[1]);
        MD[1] = MV[1];
        prefetch(pl, IV[0], MV[0], RB[0]);
        pl = next(pl);
        lookup(IV[2], MV[2], RB[2], W[2], RC[2]);
        MD[2] = MV[2];
        prefetch(pl, IV[1], MV[1], RB[1]);
        pl = next(pl);
        // step q, slot k = q % 4: decode slot k; look up slot (k + 3) % 4; load
        // position q + 6 into slot (k + 2) % 4 (looked up at step q - 1)
        auto step = [&](int q, unsigned& w_d, unsigned& m_d, uint4& c_d, unsigned& iv_w, unsigned& mv_w,
                        long long& rb_w, unsigned& w_w, unsigned& m_w, uint4& c_w, unsigned& iv_l, unsigned& mv_l,
                        long long& rb_l) {
            const int s = q % kGmStages;
            if (q >= kGmStages) {
                if (lane == 0) gm_wait(&s_empty[s], (static_cast<unsigned>(q / kGmStages) & 1u) ^ 1u, dead);
                __syncwarp();
            }
            uint4 o;
            if (m_d & 0x8000u) {  // overflow record: its coordinates, or zero past +-2048
                o = gm_far(c_d) ? make_uint4(0, 0, 0, 0) : gm_coords_f16(c_d);
            } else {
                const uint2 rbt = s_root[m_d & 0xFFu];  // R + 2 bytewise; entry 0: +2 everywhere
                const unsigned lo = (w_d & 0x0F0F0F0Fu) + rbt.x, hi = ((w_d >> 4) & 0x0F0F0F0Fu) + rbt.y;
                // fp16 1024 + (P + 10) - 1034 = P, pairs in column order
                o.x = hsub2_bits(prmt(lo, hi, 0x8480u) | 0x64006400u, 0x640A640Au);
                o.y = hsub2_bits(prmt(lo, hi, 0x8581u) | 0x64006400u, 0x640A640Au);
                o.z = hsub2_bits(prmt(lo, hi, 0x8682u) | 0x64006400u, 0x640A640Au);
                o.w = hsub2_bits(prmt(lo, hi, 0x8783u) | 0x64006400u, 0x640A640Au);
            }
            *reinterpret_cast<uint4*>(stages + s * kGmStageBytes + gm_core_off(rl, j)) = o;
            fence_proxy_async_smem();  // this thread's operand write, visible to the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_full[s]);
            lookup(iv_w, mv_w, rb_w, w_w, c_w);  // position q + 3
            m_w = mv_w;
            prefetch(pl, iv_l, mv_l, rb_l);  // position q + 6
            pl = next(pl);
            pd = next(pd);
        };
        for (int q = 0; pd.u < nunits; q += 4) {
            step(q, W[0], MD[0], RC[0], IV[3], MV[3], RB[3], W[3], MD[3], RC[3], IV[2], MV[2], RB[2]);
            if (pd.u >= nunits) break;
            step(q + 1, W[1], MD[1], RC[1], IV[0], MV[0], RB[0], W[0], MD[0], RC[0], IV[3], MV[3], RB[3]);
            if (pd.u >= nunits) break;
            step(q + 2, W[2], MD[2], RC[2], IV[1], MV[1], RB[1], W[1], MD[1], RC[1], IV[0], MV[0], RB[0]);
            if (pd.u >= nunits) break;
            step(q + 3, W[3], MD[3], RC[3], IV[2], MV[2], RB[2], W[2], MD[2], RC[2], IV[1], MV[1], RB[1]);
        }
    } else if (warp == kGmCopyWarp) {
        // ------------------------------------------------------ activation copies
        if (lane == 0) {
            int q = 0;
            for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
                const GmUnit U = gm_unit(G, u);
                const int nt = min(kGmTok, G.batch - U.tt * kGmTok);
                const unsigned bytes = static_cast<unsigned>((nt + 15) / 16 * 16) * kGmKCols * 2;
                for (int kt = U.k0; kt < U.k1; ++kt, ++q) {
                    const int s = q % kGmStages;
                    if (q >= kGmStages) gm_wait(&s_empty[s], (static_cast<unsigned>(q / kGmStages) & 1u) ^ 1u, dead);
                    mbar_arrive_expect_tx(&s_full[s], bytes);
                    bulk_load(stages + s * kGmStageBytes + kGmABytes,
                              p.img + (static_cast<size_t>(U.tt) * G.nkt + kt) * kGmBBytes, bytes, &s_full[s]);
                }
            }
            // the copies started here have landed (normally long ago): the last
            // position of each stage, q - 1 - ((q - 1 - s) mod 4)
            bool dummy = false;
            for (int s = 0; s < kGmStages; ++s) {
                const int last = q - 1 - (((q - 1 - s) % kGmStages) + kGmStages) % kGmStages;
                if (last >= 0) gm_wait(&s_full[s], static_cast<unsigned>(last / kGmStages) & 1u, dummy);
            }
        }
        __syncwarp();
    } else if (warp == kGmMmaWarp) {
        // ------------------------------------------------------ MMA issue
        if (lane == 0) {
            int q = 0, i = 0;
            for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
                const GmUnit U = gm_unit(G, u);
                const int ab = i & 1;
                if (i >= 2) gm_wait(&s_acce[ab], static_cast<unsigned>((i >> 1) - 1) & 1u, dead);  // epilogue done
                tc_fence_after_sync();
                const int nt = min(kGmTok, G.batch - U.tt * kGmTok);
                const uint32_t idesc = gm_idesc((nt + 15) / 16 * 16);
                const uint32_t d = tmem + static_cast<uint32_t>(ab * kGmTok);
                for (int kt = U.k0; kt < U.k1; ++kt, ++q) {
                    const int s = q % kGmStages;
                    gm_wait(&s_full[s], static_cast<unsigned>(q / kGmStages) & 1u, dead);
                    tc_fence_after_sync();
                    const uint32_t a0 = smem_addr(stages + s * kGmStageBytes);
                    const uint32_t b0 = a0 + kGmABytes;
#pragma unroll
                    for (int k = 0; k < 2; ++k)  // K = 16: chunks 2k and 2k + 1, 256 bytes on per step
                        umma_f16(d, gm_sdesc(a0 + 256u * k), gm_sdesc(b0 + 256u * k), idesc, kt > U.k0 || k > 0);
                    umma_commit(&s_empty[s]);
                }
                umma_commit(&s_accf[ab]);
            }
            // every MMA issued has completed before tensor memory is freed
            umma_commit(&s_done);
            bool dummy = false;
            gm_wait(&s_done, 0u, dummy);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;  // tensor-memory lanes 32 quarter .. + 31
        int i = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
            const GmUnit U = gm_unit(G, u);
            const int ab = i & 1;
            gm_wait(&s_accf[ab], static_cast<unsigned>(i >> 1) & 1u, dead);
            tc_fence_after_sync();
            const int r = U.rt * kGmRows + 32 * quarter + lane;
            const bool rok = r < G.rows;
            const int t0 = U.tt * kGmTok;
            const int nt = min(kGmTok, G.batch - t0);
            const bool direct = G.nsplit == 1;
            const float sr = rok ? 0.5f * __ldg(p.scale + r) : 0.f;
            const bool far = rok && direct && __ldcg(p.farf + r) != 0;
#pragma unroll 1
            for (int c = 0; c < nt; c += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + static_cast<uint32_t>(ab * kGmTok) + (static_cast<uint32_t>(32 * quarter) << 16) +
                              static_cast<uint32_t>(c),
                          v);
                if (!rok) continue;
                if (direct) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int t = t0 + c + k;
                        if (c + k < nt) {
                            float a = __uint_as_float(v[k]);
                            if (far) a += gm_far_sum(G, p.img, p.ovf, p.ovf_rp, p.ovf_n, p.group_base, r, t);
                            p.y[static_cast<size_t>(t) * G.rows + r] = gm_bf16(a * __ldcg(p.xe + t) * sr);
                        }
                    }
                } else {
                    float* dst = p.part + (static_cast<size_t>(U.split) * G.batch + t0 + c) * G.rows + r;
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        if (c + k < nt) dst[static_cast<size_t>(k) * G.rows] = __uint_as_float(v[k]);
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&s_acce[ab]);
        }
    }
    if (dead) atomicOr(p.err, 1ull);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kGmMmaWarp) tmem_dealloc(tmem, 2 * kGmTok);
}

// ---------------------------------------------------------------------------
// finalize (several K splits)
// ---------------------------------------------------------------------------
struct GmFinParams {
    const float* part;
    const float* xe;
    const float* scale;
    const uint8_t* farf;
    const unsigned char* img;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    long long ovf_n;
    long long group_base;
    uint16_t* y;
    GmGeom g;
};

__global__ void __launch_bounds__(256) k_gm_fin(const __grid_constant__ GmFinParams p) {
    pdl_wait();
    const GmGeom& G = p.g;
    const size_t n = static_cast<size_t>(G.batch) * G.rows;
    for (size_t e = blockIdx.x * 256ull + threadIdx.x; e < n; e += static_cast<size_t>(gridDim.x) * 256) {
        const int t = static_cast<int>(e / G.rows), r = static_cast<int>(e % G.rows);
        float a = 0.f;
        for (int s = 0; s < G.nsplit; ++s) a += __ldcs(p.part + static_cast<size_t>(s) * n + e);
        if (p.farf[r]) a += gm_far_sum(G, p.img, p.ovf, p.ovf_rp, p.ovf_n, p.group_base, r, t);
        p.y[e] = gm_bf16(a * p.xe[t] * (0.5f * p.scale[r]));
    }
}

}  // namespace e8q
