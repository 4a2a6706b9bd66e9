// K3 fast path: decode / dequantise for widths that are multiples of 256
// ("E8-QAT", abstract: the core encoding and the sparse extension keep the
// selected lattice points exactly).
//
// CTA = 7 compute warps + 1 staging warp over row tiles of up to 14,336
// elements (1,792 groups), tiles dealt round-robin.  While the compute
// warps rebuild tile k, the staging warp prepares tile k + 1 in the other
// half of two shared-memory buffers: asynchronous copies bring the tile's
// 16-bit indices, its escape records and overflow group ids (one contiguous
// range of each record array, since records are listed per row with rows in
// order) and its row scales; it then scatters the records into a map
// group -> root + 1 / 0x8000 | overflow offset.  The record ranges of
// tile k + 2 are read one iteration ahead.  One barrier per iteration; the
// only other wait is the hardware wait for the warp's own copies.
//
// Two compute layouts:
// - rotated basis, bf16(s * p) with one rounding of the exact product: lane
//   = group, 32 consecutive groups a step, so index reads, map reads and the
//   16-byte stores are contiguous; few registers, four CTAs an SM.  The
//   staging warp also fills a 32-entry table per row of bf16(s * P / 2) for
//   P = -16 .. 15 (64 bytes, one word per bank: lookups never conflict), so
//   a coordinate costs one table read; overflow groups (whose coordinates may
//   pass that range) are rewritten by the staging warp with the exact
//   products one iteration later, after the barrier;
// - original basis: each warp rebuilds one 2048-element window in the
//   layout of the fast encode's dequant (lane (a, q), row h = group
//   32 a + 4 h + q) and runs the same register Hadamard
//   (window_dequant_original); two CTAs an SM.
// Both clear the map entries they read, so a map half is empty again when
// the staging warp next fills it.  The results equal the general decode
// kernel's.
#pragma once
#include "common.cuh"
#include "encode_fast.cuh"
#include "lattice.cuh"
#include "ptx.cuh"

namespace e8q {

constexpr int kDfWarps = 7;                     // compute warps
constexpr int kDfThreads = (kDfWarps + 1) * 32;  // + the staging warp
constexpr int kDfTileElems = kDfWarps * 2048;
constexpr int kDfTileGroups = kDfTileElems / 8;
constexpr int kDfEscCap = kDfTileGroups;  // escape records staged in shared memory (a valid tile has no more)
constexpr int kDfOvfCap = 512;            // overflow group ids staged; the rest are read directly
constexpr int kDfCtasRot = 4, kDfCtasOrig = 2;
// dynamic shared memory: [transpose scratch, original basis only] index
// buffers [2], maps [2], escape staging, overflow staging
constexpr size_t kDfScratchBytes = static_cast<size_t>(kDfWarps) * 4096;
constexpr size_t kDfIdxBytes = 2 * kDfTileGroups * 2;
constexpr size_t kDfMapBytes = 2 * kDfTileGroups * 2;
constexpr size_t kDfStageBytes = kDfIdxBytes + kDfMapBytes + kDfEscCap * 8 + kDfOvfCap * 4;

__host__ __device__ constexpr size_t decode_fast_smem_bytes(bool original) {
    return (original ? kDfScratchBytes : 0) + kDfStageBytes;
}

__host__ __device__ inline int decode_fast_rows_per_tile(int cols) {
    int r = kDfTileElems / cols;
    return r < 1 ? 1 : (r > kMaxTileRows ? kMaxTileRows : r);
}

// record ranges [e0, e1) and [o0, o1) of tile t, clamped to the arrays
struct DfRange {
    long long e0, e1, o0, o1;
};

__device__ __forceinline__ DfRange df_range(const DecodeParams& p, int t) {
    DfRange r{0, 0, 0, 0};
    if (t >= p.n_tiles) return r;
    const int r0 = t * p.rpt, r1 = min(r0 + p.rpt, p.rows);
    if (p.esc_rp) {
        r.e0 = max(static_cast<long long>(__ldg(p.esc_rp + r0)), 0ll);
        r.e1 = min(static_cast<long long>(__ldg(p.esc_rp + r1)), p.esc_n);
    }
    if (p.ovf_rp) {
        r.o0 = max(static_cast<long long>(__ldg(p.ovf_rp + r0)), 0ll);
        r.o1 = min(static_cast<long long>(__ldg(p.ovf_rp + r1)), p.ovf_n);
    }
    return r;
}

struct DfShared {
    uint16_t* idx;  // [2][kDfTileGroups]
    uint16_t* map;  // [2][kDfTileGroups]
    uint2* esc;     // [kDfEscCap]
    uint32_t* og;   // [kDfOvfCap]
};

__device__ __forceinline__ DfShared df_shared(unsigned char* base) {
    DfShared s;
    s.idx = reinterpret_cast<uint16_t*>(base);
    s.map = reinterpret_cast<uint16_t*>(base + kDfIdxBytes);
    s.esc = reinterpret_cast<uint2*>(base + kDfIdxBytes + kDfMapBytes);
    s.og = reinterpret_cast<uint32_t*>(base + kDfIdxBytes + kDfMapBytes + kDfEscCap * 8);
    return s;
}

__device__ __forceinline__ void df_map_escape(uint16_t* map, uint2 rec, long long g0, int G) {
    const long long gl = static_cast<long long>(rec.x) - g0;
    const unsigned root = (rec.y >> 16) & 0xFFu;
    if (gl >= 0 && gl < G && root < 240) map[gl] = static_cast<uint16_t>(root + 1);
}

__device__ __forceinline__ void df_map_overflow(uint16_t* map, uint32_t group, long long off, long long g0, int G) {
    const long long gl = static_cast<long long>(group) - g0;
    if (gl >= 0 && gl < G && off < 0x7FFF) map[gl] = static_cast<uint16_t>(0x8000 | off);
}

// Staging warp: tile t (record ranges rg) into buffer half nb.
__device__ __forceinline__ void df_stage(const DecodeParams& p, int t, const DfRange& rg, const DfShared& sh, int nb,
                                         float* rows, float* rowm, long long* o0, float sqb, int lane,
                                         uint16_t (*lut)[32]) {
    const int r0 = t * p.rpt, nr = min(p.rpt, p.rows - r0);
    const int gpr = p.cols >> 3, G = nr * gpr;
    const long long g0 = p.group_base + static_cast<long long>(r0) * gpr;
    uint16_t* sidx = sh.idx + nb * kDfTileGroups;
    uint16_t* smap = sh.map + nb * kDfTileGroups;
    // G is a multiple of 32 and the rows start 64-byte aligned in a 16-byte
    // aligned index array: the tile's indices are whole 16-byte words
    const uint16_t* src = p.idx + static_cast<size_t>(r0) * gpr;
    for (int j = lane; j < (G >> 3); j += 32) cp_async16(sidx + 8 * j, src + 8 * j);
    const int ne = static_cast<int>(max(0ll, min(rg.e1 - rg.e0, static_cast<long long>(kDfEscCap))));
    for (int j = lane; j < ne; j += 32) cp_async8(sh.esc + j, p.esc + rg.e0 + j);
    const int no = static_cast<int>(max(0ll, min(rg.o1 - rg.o0, static_cast<long long>(kDfOvfCap))));
    for (int j = lane; j < no; j += 32) cp_async4(sh.og + j, &p.ovf[rg.o0 + j].group);
    for (int j = lane; j < nr; j += 32) cp_async4(rows + j, p.scale + r0 + j);
    cp_async_commit();
    cp_async_wait_all();
    __syncwarp();
    // escapes first, then overflows, as the general decode does
    for (int j = lane; j < ne; j += 32) df_map_escape(smap, sh.esc[j], g0, G);
    for (long long e = rg.e0 + ne + lane; e < rg.e1; e += 32)
        df_map_escape(smap, __ldg(reinterpret_cast<const uint2*>(p.esc + e)), g0, G);
    __syncwarp();
    for (int j = lane; j < no; j += 32) df_map_overflow(smap, sh.og[j], j, g0, G);
    for (long long o = rg.o0 + no + lane; o < rg.o1; o += 32) df_map_overflow(smap, __ldg(&p.ovf[o].group), o - rg.o0, g0, G);
    for (int j = lane; j < nr; j += 32) rowm[j] = rows[j] / sqb;
    if (lut) {  // rotated basis: each row's bf16(s * P / 2) for P = lane - 16
        for (int r = 0; r < nr; ++r)
            lut[r][lane] = __bfloat16_as_ushort(bf16_of_product(rows[r], 0.5f * static_cast<float>(lane - 16)));
    }
    if (lane == 0) *o0 = rg.o0;
}

// Rotated basis, after tile t's compute warps have stored it: its overflow
// groups (whose coordinates may pass the row tables' range) rewritten with
// the exact products, from the records and the global scales.
__device__ __forceinline__ void df_fix_overflow(const DecodeParams& p, int t, const DfRange& rg, int lane) {
    if (t < 0 || t >= p.n_tiles) return;
    const int r0 = t * p.rpt, nr = min(p.rpt, p.rows - r0);
    const int gpr = p.cols >> 3, G = nr * gpr;
    const long long g0 = p.group_base + static_cast<long long>(r0) * gpr;
    for (long long o = rg.o0 + lane; o < rg.o1; o += 32) {
        const e8q_overflow& rec = p.ovf[o];
        const long long gl = static_cast<long long>(__ldg(&rec.group)) - g0;
        if (gl < 0 || gl >= G) continue;
        const int row = static_cast<int>(gl / gpr);
        const float s = __ldg(p.scale + r0 + row);
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = static_cast<float>(rec.coord2[e]);
        uint4 out;
        out.x = bf16x2_of_half_products(s, v[0], v[1]);
        out.y = bf16x2_of_half_products(s, v[2], v[3]);
        out.z = bf16x2_of_half_products(s, v[4], v[5]);
        out.w = bf16x2_of_half_products(s, v[6], v[7]);
        *reinterpret_cast<uint4*>(p.out + static_cast<size_t>(r0) * p.cols + 8 * gl) = out;
    }
}

// One group's doubled coordinates from its core index and map entry.
__device__ __forceinline__ void df_point(uint2 cw, unsigned m, const e8q_overflow* ovf, long long o0, float (&v)[8]) {
    uint2 add = make_uint2(0, 0);
    if (m >= 1 && m <= 240) add = g_root8[m - 1];
    // core point + root, bytewise (every sum fits a signed byte)
    bytes_to_floats(make_uint2(__vadd4(cw.x, add.x), __vadd4(cw.y, add.y)), v);
    if (m & 0x8000u) {  // overflow record: the point itself
        const e8q_overflow& rec = ovf[o0 + (m & 0x7FFFu)];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = static_cast<float>(rec.coord2[e]);
    }
}

template <bool kOriginal>
__global__ void __launch_bounds__(kDfThreads, kOriginal ? kDfCtasOrig : kDfCtasRot)
    k_decode_fast(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float s_rows[2][kMaxTileRows], s_rowm[2][kMaxTileRows];
    __shared__ long long s_o0[2];
    __shared__ uint16_t s_lut[kOriginal ? 1 : 2][kOriginal ? 1 : kMaxTileRows][32];  // rotated: row tables
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool staging = warp == kDfWarps;
    const DfShared sh = df_shared(smem + (kOriginal ? kDfScratchBytes : 0));
    const int C = p.cols, gpr = C >> 3;
    const float sqb = sqrtf(static_cast<float>(1 << p.logb));
    // both maps start empty; afterwards every entry set is cleared by the warp that reads it
    for (int i = tid; i < kDfTileGroups; i += kDfThreads) reinterpret_cast<uint32_t*>(sh.map)[i] = 0u;
    DfRange next{0, 0, 0, 0}, staged1{0, 0, 0, 0}, staged2{0, 0, 0, 0};  // ranges staged 1 and 2 iterations ago
    if (staging) next = df_range(p, blockIdx.x);
    __syncthreads();

    // iteration k: compute warps rebuild tile t = blockIdx + k * grid from
    // buffer half k & 1 while the staging warp fills the other half with the
    // CTA's next tile
    for (int k = -1;; ++k) {
        const int t = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
        if (t >= p.n_tiles) break;
        const int tn = t + static_cast<int>(gridDim.x);
        if (staging) {
            // rotated basis: the tile computed in the previous iteration gets its overflow groups
            if (!kOriginal) df_fix_overflow(p, t - static_cast<int>(gridDim.x), staged2, lane);
            DfRange cur{0, 0, 0, 0};
            if (tn < p.n_tiles) {
                const int nb = (k + 1) & 1;
                cur = next;
                next = df_range(p, tn + static_cast<int>(gridDim.x));
                df_stage(p, tn, cur, sh, nb, s_rows[nb], s_rowm[nb], &s_o0[nb], sqb, lane,
                         kOriginal ? nullptr : s_lut[kOriginal ? 0 : nb]);
            }
            staged2 = staged1;
            staged1 = cur;
        } else if (t >= 0) {
            const int b = k & 1;
            const int r0 = t * p.rpt;
            const int nr = min(p.rpt, p.rows - r0);
            const int n = nr * C, G = nr * gpr;
            const uint16_t* ti = sh.idx + b * kDfTileGroups;
            uint16_t* tm = sh.map + b * kDfTileGroups;
            const long long o0 = s_o0[b];
            uint16_t* dq = p.out + static_cast<size_t>(r0) * C;
            const int w = warp;
            if (!kOriginal) {
                // lane = group: 8 steps of 32 consecutive groups, each step inside one row
                const int gw = 256 * w;
                const int steps = max(0, min(8, (G - gw) >> 5));
                uint2 cw[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) cw[j] = j < steps ? __ldg(g_core8 + ti[gw + 32 * j + lane]) : make_uint2(0, 0);
                int row = gw / gpr, rem = gw - row * gpr;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j >= steps) break;
                    const int g = gw + 32 * j + lane;
                    const unsigned m = tm[g];
                    if (m) tm[g] = 0;
                    // core point + root bytewise (|P| <= 8); an overflow group stores the
                    // core point of index 0 here and is rewritten after the barrier
                    uint2 add = make_uint2(0, 0);
                    if (m >= 1 && m <= 240) add = g_root8[m - 1];
                    const unsigned w0 = __vadd4(cw[j].x, add.x), w1 = __vadd4(cw[j].y, add.y);
                    const unsigned i0 = (w0 & 0x1F1F1F1Fu) ^ 0x10101010u, i1 = (w1 & 0x1F1F1F1Fu) ^ 0x10101010u;  // P + 16
                    const uint16_t* lt = s_lut[kOriginal ? 0 : b][row];
                    uint4 o;
                    o.x = static_cast<unsigned>(lt[i0 & 0xFFu]) | (static_cast<unsigned>(lt[(i0 >> 8) & 0xFFu]) << 16);
                    o.y = static_cast<unsigned>(lt[(i0 >> 16) & 0xFFu]) | (static_cast<unsigned>(lt[i0 >> 24]) << 16);
                    o.z = static_cast<unsigned>(lt[i1 & 0xFFu]) | (static_cast<unsigned>(lt[(i1 >> 8) & 0xFFu]) << 16);
                    o.w = static_cast<unsigned>(lt[(i1 >> 16) & 0xFFu]) | (static_cast<unsigned>(lt[i1 >> 24]) << 16);
                    *reinterpret_cast<uint4*>(dq + 8 * g) = o;
                    rem += 32;
                    if (rem >= gpr) {
                        rem -= gpr;
                        ++row;
                    }
                }
            } else {
                const int nwin = (n + 2047) >> 11;
                if (w < nwin) {
                    const int wbase = 2048 * w;
                    const int nchunks = max(0, min(8, (n - wbase) >> 8));
                    const int a = lane >> 2, q = lane & 3;
                    const bool lane_ok = a < nchunks;
                    float v[8][8];
                    uint2 cw[8];
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const int gt = 256 * w + 32 * a + 4 * h + q;
                        cw[h] = (lane_ok && gt < G) ? __ldg(g_core8 + ti[gt]) : make_uint2(0, 0);
                    }
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const int gt = 256 * w + 32 * a + 4 * h + q;
                        const unsigned m = (lane_ok && gt < G) ? tm[gt] : 0u;
                        if (m) tm[gt] = 0;
                        df_point(cw[h], m, p.ovf, o0, v[h]);
                    }
                    const bool win_rows = (C & 2047) == 0;
                    const HFrag hf = make_hfrag(lane);
                    float4* scratch = reinterpret_cast<float4*>(smem + warp * 4096);
                    window_dequant_original(v, scratch, lane, hf, p.logb, dq, p.signs, C, wbase, nchunks, s_rowm[b],
                                            win_rows, win_rows ? (wbase / C) : 0);
                }
            }
        }
        __syncthreads();
    }
    // rotated basis: the CTA's last tile gets its overflow groups
    if (!kOriginal && staging) {
        const int nt = static_cast<int>(blockIdx.x) < p.n_tiles
                           ? (p.n_tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x)
                           : -1;
        df_fix_overflow(p, static_cast<int>(blockIdx.x) + nt * static_cast<int>(gridDim.x), staged2, lane);
    }
}

}  // namespace e8q
