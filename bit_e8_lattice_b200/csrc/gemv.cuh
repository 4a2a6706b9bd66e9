// K4 + K5: dequant-GEMV from the 2-bit form ("E8-QAT", abstract: decoding
// throughput of the 2-bit representation).
//
//   y[b][r] = s_r / 2 * ( sum_g <P_core[idx_rg], xr_bg>
//                       + sum_{escapes of row r} <R_root, xr_bg>
//                       + sum_{overflows of row r} <P_record, xr_bg> ),
//   xr_b = H_B (d (.) x_b) / sqrt(B)   (blockwise, fp32),
// which equals sum_c w~[r][c] x[b][c] with w~ the original-basis weights.
#pragma once
#include "common.cuh"
#include "lattice.cuh"

namespace e8q {

constexpr int kRhtThreads = 256;
constexpr int kGemvThreads = 256;

struct RhtParams {
    const uint16_t* x;  // bf16 [batch][cols]
    const int8_t* signs;
    float* xr;          // fp32 [batch][cols]
    int32_t cols;
    int32_t logb;
};

__global__ void __launch_bounds__(kRhtThreads) k_rht_x(const __grid_constant__ RhtParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* buf = reinterpret_cast<float*>(smem);
    const int b = blockIdx.x, C = p.cols;
    const uint16_t* xb = p.x + static_cast<size_t>(b) * C;
    for (int c = threadIdx.x; c < C; c += kRhtThreads) {
        const float v = __uint_as_float(static_cast<unsigned>(xb[c]) << 16);
        buf[c] = p.signs[c] < 0 ? -v : v;
    }
    __syncthreads();
    if (p.logb > 0) fwht_smem(buf, C, p.logb);
    const float inv = 1.0f / sqrtf(static_cast<float>(1 << p.logb));
    for (int c = threadIdx.x; c < C; c += kRhtThreads) p.xr[static_cast<size_t>(b) * C + c] = buf[c] * inv;
}

struct GemvParams {
    const uint16_t* idx;
    const float* scale;
    const e8q_escape* esc;
    const int64_t* esc_rp;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    const float* xr;  // fp32 [batch][cols]
    uint16_t* y;      // bf16 [batch][rows]
    long long esc_n;
    long long ovf_n;
    long long group_base;
    int32_t rows;
    int32_t cols;
    int32_t batch;
};

__global__ void __launch_bounds__(kGemvThreads) k_gemv(const __grid_constant__ GemvParams p) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (kGemvThreads / 32);
    const int C = p.cols, gpr = C >> 3;
    for (int r = blockIdx.x * (kGemvThreads / 32) + (threadIdx.x >> 5); r < p.rows; r += warps) {
        const float s = p.scale[r];
        const size_t g0 = static_cast<size_t>(r) * gpr;
        for (int bc = 0; bc < p.batch; bc += 8) {
            const int nb = min(8, p.batch - bc);
            float acc[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[b] = 0.f;
            for (int g = lane; g < gpr; g += 32) {
                const uint2 cw = g_core8[p.idx[g0 + g]];
                float P[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) P[i] = coord_of(cw, i);
#pragma unroll
                for (int b = 0; b < 8; ++b)
                    if (b < nb) {
                        const float4* x = reinterpret_cast<const float4*>(p.xr + static_cast<size_t>(bc + b) * C) + 2 * g;
                        const float4 u = x[0], v = x[1];
                        acc[b] = fmaf(P[0], u.x, fmaf(P[1], u.y, fmaf(P[2], u.z, fmaf(P[3], u.w, acc[b]))));
                        acc[b] = fmaf(P[4], v.x, fmaf(P[5], v.y, fmaf(P[6], v.z, fmaf(P[7], v.w, acc[b]))));
                    }
            }
            if (p.esc_rp) {
                const long long e1 = min(static_cast<long long>(p.esc_rp[r + 1]), p.esc_n);
                for (long long e = max(static_cast<long long>(p.esc_rp[r]), 0ll) + lane; e < e1; e += 32) {
                    const e8q_escape rec = p.esc[e];
                    const long long gl = static_cast<long long>(rec.group) - p.group_base - static_cast<long long>(g0);
                    if (gl < 0 || gl >= gpr || rec.root >= 240) continue;
                    const uint2 rw = g_root8[rec.root];
#pragma unroll
                    for (int b = 0; b < 8; ++b)
                        if (b < nb) {
                            const float* x = p.xr + static_cast<size_t>(bc + b) * C + 8 * gl;
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[b] = fmaf(static_cast<float>(coord_of(rw, i)), x[i], acc[b]);
                        }
                }
            }
            if (p.ovf_rp) {
                const long long o1 = min(static_cast<long long>(p.ovf_rp[r + 1]), p.ovf_n);
                for (long long o = max(static_cast<long long>(p.ovf_rp[r]), 0ll) + lane; o < o1; o += 32) {
                    const e8q_overflow rec = p.ovf[o];
                    const long long gl = static_cast<long long>(rec.group) - p.group_base - static_cast<long long>(g0);
                    if (gl < 0 || gl >= gpr) continue;
#pragma unroll
                    for (int b = 0; b < 8; ++b)
                        if (b < nb) {
                            const float* x = p.xr + static_cast<size_t>(bc + b) * C + 8 * gl;
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[b] = fmaf(static_cast<float>(rec.coord2[i]), x[i], acc[b]);
                        }
                }
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc[b] += __shfl_xor_sync(0xFFFFFFFFu, acc[b], off);
            }
            if (lane < nb) {
                float v = acc[0];
#pragma unroll
                for (int b = 1; b < 8; ++b)
                    if (lane == b) v = acc[b];
                p.y[static_cast<size_t>(bc + lane) * p.rows + r] = __bfloat16_as_ushort(__float2bfloat16_rn(0.5f * s * v));
            }
        }
    }
}

}  // namespace e8q
