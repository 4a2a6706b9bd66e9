// K3: decode / dequantise ("E8-QAT", abstract: the core encoding and the
// sparse extension keep the selected lattice points exactly).
//
// Per row tile: p = core[idx] for every group, the row's escape records
// add their root and overflow records replace the point, then either
// bf16(s * p) (Hadamard domain, one rounding of the exact product) or
// bf16(d (.) H_B (s * p) / sqrt(B)) (original basis).
#pragma once
#include "common.cuh"
#include "lattice.cuh"

namespace e8q {

constexpr int kDecThreads = 256;

struct DecodeParams {
    const uint16_t* idx;
    const float* scale;
    const int8_t* signs;
    const e8q_escape* esc;
    const int64_t* esc_rp;
    const e8q_overflow* ovf;
    const int64_t* ovf_rp;
    uint16_t* out;
    long long esc_n;
    long long ovf_n;
    long long group_base;
    int32_t rows;
    int32_t cols;
    int32_t logb;
    int32_t basis;
    int32_t rpt;
    int32_t n_tiles;
};

__global__ void __launch_bounds__(kDecThreads) k_decode(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* tile = reinterpret_cast<float*>(smem);  // doubled coordinates, then values
    const int tid = threadIdx.x;
    const int C = p.cols, gpr = C >> 3;
    const float B = static_cast<float>(1 << p.logb);
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
        const int r0 = t * p.rpt;
        const int nr = min(p.rpt, p.rows - r0);
        const int n = nr * C, G = nr * gpr;
        const size_t g0 = static_cast<size_t>(r0) * gpr;
        for (int g = tid; g < G; g += kDecThreads) {
            const uint2 cw = g_core8[p.idx[g0 + g]];
            float4* dst = reinterpret_cast<float4*>(tile) + 2 * g;
            dst[0] = make_float4(coord_of(cw, 0), coord_of(cw, 1), coord_of(cw, 2), coord_of(cw, 3));
            dst[1] = make_float4(coord_of(cw, 4), coord_of(cw, 5), coord_of(cw, 6), coord_of(cw, 7));
        }
        __syncthreads();
        if (p.esc_rp) {
            const long long e0 = max(static_cast<long long>(p.esc_rp[r0]), 0ll), e1 = min(static_cast<long long>(p.esc_rp[r0 + nr]), p.esc_n);
            for (long long e = e0 + tid; e < e1; e += kDecThreads) {
                const e8q_escape rec = p.esc[e];
                const long long gl = static_cast<long long>(rec.group) - p.group_base - static_cast<long long>(g0);
                if (gl < 0 || gl >= G || rec.root >= 240) continue;  // not this tile's: ignore
                const uint2 rw = g_root8[rec.root];
#pragma unroll
                for (int i = 0; i < 8; ++i) tile[8 * gl + i] += coord_of(rw, i);
            }
        }
        if (p.ovf_rp) {
            const long long o0 = max(static_cast<long long>(p.ovf_rp[r0]), 0ll), o1 = min(static_cast<long long>(p.ovf_rp[r0 + nr]), p.ovf_n);
            for (long long o = o0 + tid; o < o1; o += kDecThreads) {
                const e8q_overflow rec = p.ovf[o];
                const long long gl = static_cast<long long>(rec.group) - p.group_base - static_cast<long long>(g0);
                if (gl < 0 || gl >= G) continue;
#pragma unroll
                for (int i = 0; i < 8; ++i) tile[8 * gl + i] = rec.coord2[i];
            }
        }
        __syncthreads();
        uint4* out = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(r0) * C);
        if (p.basis == E8Q_DEQUANT_ROTATED) {
            for (int q = tid; q < (n >> 3); q += kDecThreads) {
                const float s = p.scale[r0 + q / gpr];
                const float4 a = reinterpret_cast<const float4*>(tile)[2 * q];
                const float4 b = reinterpret_cast<const float4*>(tile)[2 * q + 1];
                out[q] = make_uint4(pack_bf16x2(bf16_of_product(s, 0.5f * a.x), bf16_of_product(s, 0.5f * a.y)),
                                    pack_bf16x2(bf16_of_product(s, 0.5f * a.z), bf16_of_product(s, 0.5f * a.w)),
                                    pack_bf16x2(bf16_of_product(s, 0.5f * b.x), bf16_of_product(s, 0.5f * b.y)),
                                    pack_bf16x2(bf16_of_product(s, 0.5f * b.z), bf16_of_product(s, 0.5f * b.w)));
            }
        } else {
            for (int q = tid; q < (n >> 3); q += kDecThreads) {  // p = P / 2, exact
                float4* v = reinterpret_cast<float4*>(tile) + 2 * q;
                float4 a = v[0], b = v[1];
                a.x *= 0.5f; a.y *= 0.5f; a.z *= 0.5f; a.w *= 0.5f;
                b.x *= 0.5f; b.y *= 0.5f; b.z *= 0.5f; b.w *= 0.5f;
                v[0] = a;
                v[1] = b;
            }
            __syncthreads();
            if (p.logb > 0) fwht_smem(tile, n, p.logb);  // H(p): exact in fp32
            for (int q = tid; q < (n >> 3); q += kDecThreads) {
                const int c0 = (q << 3) % C;
                const float inv = p.scale[r0 + q / gpr] / sqrtf(B);
                const uint2 dv = *reinterpret_cast<const uint2*>(p.signs + c0);
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
                out[q] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                    pack_bf16x2(o[6], o[7]));
            }
        }
        __syncthreads();
    }
}

}  // namespace e8q
