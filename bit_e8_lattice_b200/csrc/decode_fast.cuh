// K3 fast path: decode / dequantise for widths that are multiples of 256
// with an RHT block of 256..2048 ("E8-QAT", abstract: the core encoding
// and the sparse extension keep the selected lattice points exactly).
//
// CTA = 7 warps over row tiles of up to 14,336 elements, two CTAs an SM.
// The tile's escape and overflow records are one contiguous range of each record
// array (records are listed per row, rows in order): the CTA scatters them
// into a shared-memory map group -> root + 1 / overflow record.  Each warp
// then rebuilds one 2048-element window of doubled coordinates, in the
// layout the fast encode's dequant uses (lane (a, q), row h = group
// 32 a + 4 h + q), from the core table, the map and the records, and
// writes either bf16(s * p) (rotated basis, one rounding of the exact
// product) or the original basis through the same register Hadamard as the
// encode (window_dequant_original).  The results equal the general
// decode kernel's.
#pragma once
#include "common.cuh"
#include "encode_fast.cuh"
#include "lattice.cuh"

namespace e8q {

constexpr int kDfWarps = 7;
constexpr int kDfThreads = kDfWarps * 32;
constexpr int kDfTileElems = kDfWarps * 2048;
constexpr int kDfTileGroups = kDfTileElems / 8;
constexpr size_t kDfSmemBytes = static_cast<size_t>(kDfWarps) * 4096;  // transpose scratch per warp

__host__ __device__ inline int decode_fast_rows_per_tile(int cols) {
    int r = kDfTileElems / cols;
    return r < 1 ? 1 : (r > kMaxTileRows ? kMaxTileRows : r);
}

__global__ void __launch_bounds__(kDfThreads, 2) k_decode_fast(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ uint16_t s_map[kDfTileGroups];  // 0, root + 1, or 0x8000 | overflow offset in the tile
    __shared__ float s_rows[kMaxTileRows], s_rowm[kMaxTileRows];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = p.cols, gpr = C >> 3;
    const float sqb = sqrtf(static_cast<float>(1 << p.logb));
    const HFrag hf = make_hfrag(lane);
    float4* scratch = reinterpret_cast<float4*>(smem + warp * 4096);
    const bool win_rows = (C & 2047) == 0;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
        const int r0 = t * p.rpt;
        const int nr = min(p.rpt, p.rows - r0);
        const int n = nr * C, G = nr * gpr;
        const long long g0 = p.group_base + static_cast<long long>(r0) * gpr;
        for (int i = tid; i < G; i += kDfThreads) s_map[i] = 0;
        if (tid < nr) {
            const float s = p.scale[r0 + tid];
            s_rows[tid] = s;
            s_rowm[tid] = s / sqb;
        }
        long long o0 = 0;
        __syncthreads();
        if (p.esc_rp) {
            const long long e0 = max(static_cast<long long>(p.esc_rp[r0]), 0ll);
            const long long e1 = min(static_cast<long long>(p.esc_rp[r0 + nr]), p.esc_n);
            for (long long e = e0 + tid; e < e1; e += kDfThreads) {
                const uint2 rec = __ldg(reinterpret_cast<const uint2*>(p.esc + e));
                const long long gl = static_cast<long long>(rec.x) - g0;
                const unsigned root = (rec.y >> 16) & 0xFFu;
                if (gl >= 0 && gl < G && root < 240) s_map[gl] = static_cast<uint16_t>(root + 1);
            }
        }
        if (p.ovf_rp) {
            o0 = max(static_cast<long long>(p.ovf_rp[r0]), 0ll);
            const long long o1 = min(static_cast<long long>(p.ovf_rp[r0 + nr]), p.ovf_n);
            for (long long o = o0 + tid; o < o1; o += kDfThreads) {
                const long long gl = static_cast<long long>(__ldg(&p.ovf[o].group)) - g0;
                if (gl >= 0 && gl < G && o - o0 < 0x7FFF) s_map[gl] = static_cast<uint16_t>(0x8000 | (o - o0));
            }
        }
        __syncthreads();

        const int nwin = (n + 2047) >> 11;
        if (warp < nwin) {
            const int w = warp, wbase = 2048 * w;
            const int nchunks = max(0, min(8, (n - wbase) >> 8));
            const int a = lane >> 2, q = lane & 3;
            const bool lane_ok = a < nchunks;
            float v[8][8];
            uint2 cw[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const int gt = 256 * w + 32 * a + 4 * h + q;
                cw[h] = (lane_ok && gt < G) ? __ldg(g_core8 + p.idx[static_cast<size_t>(r0) * gpr + gt]) : make_uint2(0, 0);
            }
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const int gt = 256 * w + 32 * a + 4 * h + q;
                const unsigned m = (lane_ok && gt < G) ? s_map[gt] : 0u;
                uint2 add = make_uint2(0, 0);
                if (m >= 1 && m <= 240) add = g_root8[m - 1];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[h][e] = static_cast<float>(coord_of(cw[h], e) + coord_of(add, e));
                if (m & 0x8000u) {  // overflow record: the point itself
                    const e8q_overflow& rec = p.ovf[o0 + (m & 0x7FFFu)];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[h][e] = static_cast<float>(rec.coord2[e]);
                }
            }
            uint16_t* dq = p.out + static_cast<size_t>(r0) * C;
            const int row_w = win_rows ? (wbase / C) : 0;
            if (p.basis == E8Q_DEQUANT_ORIGINAL) {
                window_dequant_original(v, scratch, lane, hf, p.logb, dq, p.signs, C, wbase, nchunks, s_rowm, win_rows,
                                        row_w);
            } else {
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const int gt = 256 * w + 32 * a + 4 * h + q;
                    if (!lane_ok || gt >= G) continue;
                    const float s = s_rows[gt / gpr];
                    uint4 o;
                    o.x = pack_bf16x2(bf16_of_product(s, 0.5f * v[h][0]), bf16_of_product(s, 0.5f * v[h][1]));
                    o.y = pack_bf16x2(bf16_of_product(s, 0.5f * v[h][2]), bf16_of_product(s, 0.5f * v[h][3]));
                    o.z = pack_bf16x2(bf16_of_product(s, 0.5f * v[h][4]), bf16_of_product(s, 0.5f * v[h][5]));
                    o.w = pack_bf16x2(bf16_of_product(s, 0.5f * v[h][6]), bf16_of_product(s, 0.5f * v[h][7]));
                    *reinterpret_cast<uint4*>(dq + 8 * gt) = o;
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace e8q
