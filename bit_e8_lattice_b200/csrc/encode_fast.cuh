// K1 fast path: RHT + row scale + E8 projection + core encoding + ordered
// records (+ dequantised output) for bf16 weights whose width is a multiple
// of 256 and whose RHT block is 256..2048 ("E8-QAT", Figure 2 (a)-(c)).
//
// CTA = 14 compute warps + 1 service warp (128 registers a thread), persistent
// over row tiles of up to 28,672 elements (two 14336-wide rows, seven
// 4096-wide rows) taken from an atomic ticket; one barrier per iteration.
//   service warp, iteration i: claims tile i+1 and prefetches it with a
//     1-D bulk copy (TMA engine) into the other shared-memory buffer; forms
//     the chunk prefix of tile i-1's record counts, publishes them and
//     stores its 16-bit indices with a bulk copy; places tile i-2 among all
//     earlier tiles' records (decoupled look-back, bounded waits); computes
//     tile i+1's row scales from its input (the RHT is orthonormal).
//   compute warps: one 2048-element window each of tile i.  Hadamard in
//     registers: bits {0,1,3,4} of the element index by one bf16 m16n8k16
//     tensor-core MMA against H_16 straight from the (sign-flipped) bf16
//     input, bit 2 and bits 8..10 as fp32 butterflies, then an in-warp
//     transpose through shared memory and bits 5..7.  Projection and core
//     rank in registers (rank table T1 read through L1, T2 in shared
//     memory); a group outside the core takes its encoding from the escape
//     lookup table (the lane's 8 groups' gathers issued together).  Each
//     warp counts and indexes its own window and emits its own chunks of
//     tile i-3's records.
// Record order, CSR and results are the same as the generic kernel's.
#pragma once
#include "common.cuh"
#include "encode.cuh"
#include "lattice.cuh"
#include "ptx.cuh"

namespace e8q {

constexpr int kFastWarps = 14;
constexpr int kFastThreads = (kFastWarps + 1) * 32;  // compute warps, service warp
constexpr int kFastTileElems = kFastWarps * 2048;    // 28672: two 14336-wide rows, seven 4096-wide rows
constexpr int kFastTileGroups = kFastTileElems / 8;
constexpr int kFastChunks = kFastTileGroups / 32;    // 32-group chunks per tile
constexpr int kFastCnt = kFastChunks + 1;            // per record kind: chunk counts (then prefixes), total
constexpr int kFastMaxCtas = 160;
constexpr int kWaitLimit = 1 << 24;

__host__ __device__ inline int fast_rows_per_tile(int cols) {
    int r = kFastTileElems / cols;
    return r < 1 ? 1 : (r > kMaxTileRows ? kMaxTileRows : r);
}

// Pipeline depth: a tile's map, chunk counts and overflow scratch live for
// four iterations (computed, counted, placed, emitted).
constexpr int kFastSlots = 4;

// shared-memory layout (bytes)
constexpr int kFsIn = 0;                                              // bf16 [2][16384]
constexpr int kFsT2 = kFsIn + 2 * kFastTileElems * 2;                 // T1 (67 KB) is read through L1
constexpr int kFsMap = kFsT2 + kEncT2Bytes;                           // u32 [4][2048]
constexpr int kFsChunk = kFsMap + kFastSlots * kFastTileGroups * 4;   // u32 [4][2][kFastCnt]
constexpr int kFastSmemBytes = kFsChunk + kFastSlots * 2 * kFastCnt * 4 + 8;

struct FastTile {
    int t;        // ticket (>= n_tiles: none)
    int mat;
    int r0;
    int nr;
    unsigned ne;  // escape records of the tile
    unsigned no;  // overflow records of the tile
};

// ---------------------------------------------------------------- helpers
// Position of a tile group's entry in the per-tile map: the projection
// writes groups 32a + 4h + q (lane a, q; row h) together and the emission
// reads 32 consecutive groups together; xor-ing bits 2..4 with bits 5..7
// keeps both free of shared-memory bank conflicts.
__device__ __forceinline__ int map_slot(int g) { return g ^ (((g >> 5) & 7) << 2); }

__device__ __forceinline__ void bfly(float& a, float& b) {
    const float x = a;
    a = x + b;
    b = x - b;
}

__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
    const float2 a = make_float2(a0, a1), b = make_float2(b0, b1);
    const float2 s = __fadd2_rn(a, b);
    const float2 d = __ffma2_rn(b, make_float2(-1.f, -1.f), a);
    a0 = s.x; a1 = s.y; b0 = d.x; b1 = d.y;
}

// butterflies between the 8-value rows v[k] and v[k ^ m] for register bit m
template <int M>
__device__ __forceinline__ void stage_rows(float (&v)[8][8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if ((k & M) == 0)
#pragma unroll
            for (int e = 0; e < 8; e += 2) bfly2(v[k][e], v[k][e + 1], v[k + M][e], v[k + M][e + 1]);
}

// butterflies between element e and e + 4 of every row (element bit 2)
__device__ __forceinline__ void stage_e2(float (&v)[8][8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        bfly2(v[k][0], v[k][1], v[k][4], v[k][5]);
        bfly2(v[k][2], v[k][3], v[k][6], v[k][7]);
    }
}

// Swap lane bits 2..4 with the register row index (8x8 blocks of 8 values)
// through a 4 KB shared-memory region, two rounds of four values; the slot
// function keeps every 128-bit store and load phase free of bank conflicts.
__device__ __forceinline__ void warp_transpose(float (&v)[8][8], float4* scratch, int lane) {
    const int a = lane >> 2, q = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int s = 8 * (4 * k + (a >> 1)) + 2 * q + ((a ^ k) & 1);
            scratch[s] = make_float4(v[k][4 * half], v[k][4 * half + 1], v[k][4 * half + 2], v[k][4 * half + 3]);
        }
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            const int s = 8 * (4 * a + (h >> 1)) + 2 * q + ((h ^ a) & 1);
            const float4 t = scratch[s];
            v[h][4 * half] = t.x;
            v[h][4 * half + 1] = t.y;
            v[h][4 * half + 2] = t.z;
            v[h][4 * half + 3] = t.w;
        }
        __syncwarp();
    }
}

// sign flip of 8 bf16 values held as 4 packed pairs, from 8 int8 signs
__device__ __forceinline__ void apply_signs(unsigned (&r)[4], uint2 dv) {
    r[0] ^= prmt(dv.x, 0u, 0x1404u) & 0x80008000u;
    r[1] ^= prmt(dv.x, 0u, 0x3424u) & 0x80008000u;
    r[2] ^= prmt(dv.y, 0u, 0x1404u) & 0x80008000u;
    r[3] ^= prmt(dv.y, 0u, 0x3424u) & 0x80008000u;
}

__device__ __forceinline__ unsigned bf16_pm1(int neg) { return neg ? 0xBF80u : 0x3F80u; }

struct HFrag {  // B fragments of H_16 for the two n-halves
    unsigned b10, b11, b20, b21;
};

__device__ __forceinline__ HFrag make_hfrag(int lane) {
    const int g = lane >> 2, q = lane & 3;
    auto h = [](int k, int n) { return __popc(k & n) & 1; };
    HFrag f;
    f.b10 = bf16_pm1(h(2 * q, g)) | (bf16_pm1(h(2 * q + 1, g)) << 16);
    f.b11 = bf16_pm1(h(2 * q + 8, g)) | (bf16_pm1(h(2 * q + 9, g)) << 16);
    f.b20 = bf16_pm1(h(2 * q, g + 8)) | (bf16_pm1(h(2 * q + 1, g + 8)) << 16);
    f.b21 = bf16_pm1(h(2 * q + 8, g + 8)) | (bf16_pm1(h(2 * q + 9, g + 8)) << 16);
    return f;
}

// H_16 over element bits {0,1} and lane bits {0,1} of one row of 8 values
// given as packed bf16 pairs (R0 = e0,e1 ... R3 = e6,e7).
__device__ __forceinline__ void mma_h16(float (&o)[8], unsigned r0, unsigned r1, unsigned r2, unsigned r3,
                                        const HFrag& f) {
    float d1[4], d2[4];
    mma_bf16_m16n8k16(d1, r0, r2, r1, r3, f.b10, f.b11);
    mma_bf16_m16n8k16(d2, r0, r2, r1, r3, f.b20, f.b21);
    o[0] = d1[0]; o[1] = d1[1]; o[4] = d1[2]; o[5] = d1[3];
    o[2] = d2[0]; o[3] = d2[1]; o[6] = d2[2]; o[7] = d2[3];
}

// Forward transform of one window (8 chunks of 256 elements).  On return
// v is in the transposed layout: lane (a, q), row h hold the group
// g = 32 a + 4 h + q of the window.  Returns the lane's sum of squares.
__device__ __forceinline__ float window_forward(float (&v)[8][8], const unsigned (&raw)[8][4], int logb, int nchunks,
                                                float4* scratch, int lane, const HFrag& hf) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k < nchunks) {
            mma_h16(v[k], raw[k][0], raw[k][1], raw[k][2], raw[k][3], hf);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[k][e] = 0.f;
        }
    }
    stage_e2(v);
    if (logb >= 9) stage_rows<1>(v);
    if (logb >= 10) stage_rows<2>(v);
    if (logb >= 11) stage_rows<4>(v);
    warp_transpose(v, scratch, lane);
    stage_rows<1>(v);
    stage_rows<2>(v);
    stage_rows<4>(v);
    float2 ss = make_float2(0.f, 0.f);
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float2 t = make_float2(v[h][e], v[h][e + 1]);
            ss = __ffma2_rn(t, t, ss);
        }
    return ss.x + ss.y;
}

__device__ __forceinline__ void load_window_raw(unsigned (&raw)[8][4], const uint16_t* src_smem_or_global,
                                                bool from_global, const int8_t* signs, int cols, int col0, int nchunks,
                                                int lane, unsigned& nonfinite) {
    int c = (col0 + 8 * lane) % cols;  // column of this lane's first element; chunks step 256
#pragma unroll
    for (int k = 0; k < 8; ++k, c = (c + 256 >= cols) ? c + 256 - cols : c + 256) {
        if (k < nchunks) {
            const uint16_t* p = src_smem_or_global + 256 * k + 8 * lane;
            uint4 q;
            if (from_global) q = __ldg(reinterpret_cast<const uint4*>(p));
            else q = *reinterpret_cast<const uint4*>(p);
            raw[k][0] = q.x; raw[k][1] = q.y; raw[k][2] = q.z; raw[k][3] = q.w;
            if (from_global) {  // slow path: non-finite values read as 0
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const unsigned x = raw[k][j];
                    unsigned keep = 0xFFFFFFFFu;
                    if ((x & 0x7F80u) == 0x7F80u) { keep &= 0xFFFF0000u; ++nonfinite; }
                    if ((x & 0x7F800000u) == 0x7F800000u) { keep &= 0x0000FFFFu; ++nonfinite; }
                    raw[k][j] = x & keep;
                }
            }
            apply_signs(raw[k], __ldg(reinterpret_cast<const uint2*>(signs + c)));
        } else {
            raw[k][0] = raw[k][1] = raw[k][2] = raw[k][3] = 0u;
        }
    }
}

// Copy of a window from global memory to shared memory with every
// non-finite value replaced by 0 (and counted).
__device__ __forceinline__ void sanitize_window(uint16_t* dst, const uint16_t* src, int nchunks, int lane,
                                                unsigned& nonfinite) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k >= nchunks) break;
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + 256 * k + 8 * lane));
        unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            unsigned keep = 0xFFFFFFFFu;
            if ((w[j] & 0x7F80u) == 0x7F80u) { keep &= 0xFFFF0000u; ++nonfinite; }
            if ((w[j] & 0x7F800000u) == 0x7F800000u) { keep &= 0x0000FFFFu; ++nonfinite; }
            w[j] &= keep;
        }
        *reinterpret_cast<uint4*>(dst + 256 * k + 8 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Original-basis dequant of one window, in place of its lattice points:
// v holds doubled coordinates P in the transposed layout (lane (a, q), row
// h = group 32 a + 4 h + q of the window); writes bf16 (s_r / sqrt(B)) *
// d (.) H_B(p) for the window's chunks (dq_tile: the tile's first element;
// rowm[r] = s_r / sqrt(B) per tile row).  H(p) is exact.
// big_hint: 1 if the lane may hold some |P| > 255 (a superset is fine: it
// only selects the exact three-term path), 0 if it holds none, -1 to test
// the values here.
__device__ __forceinline__ void window_dequant_original(float (&v)[8][8], float4* scratch, int lane, const HFrag& hf,
                                                        int logb, uint16_t* dq_tile, const int8_t* signs, int C,
                                                        int wbase, int nchunks, const float* rowm, bool win_rows,
                                                        int row_w, int big_hint = -1) {
    // H(p) exactly: tensor-core stage on bf16 p = P/2 (split in two
    // bf16 terms when some |P| >= 256), fp32 butterflies for the rest.
    bool big = big_hint > 0;
    if (big_hint < 0) {
#pragma unroll
        for (int h = 0; h < 8; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) big |= fabsf(v[h][e]) > 255.f;
    }
    big = __any_sync(0xFFFFFFFFu, big);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        float o[8];
        unsigned r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 t = __floats2bfloat162_rn(0.5f * v[h][2 * j], 0.5f * v[h][2 * j + 1]);
            r[j] = *reinterpret_cast<const unsigned*>(&t);
        }
        mma_h16(o, r[0], r[1], r[2], r[3], hf);
        if (big) {  // p = t0 + t1 + t2, each term exact in bf16 (24 bits)
            float rem[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&r[j]);
                rem[2 * j] = 0.5f * v[h][2 * j] - __bfloat162float(hi.x);
                rem[2 * j + 1] = 0.5f * v[h][2 * j + 1] - __bfloat162float(hi.y);
            }
#pragma unroll
            for (int term = 0; term < 2; ++term) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __nv_bfloat162 t = __floats2bfloat162_rn(rem[2 * j], rem[2 * j + 1]);
                    r[j] = *reinterpret_cast<const unsigned*>(&t);
                    rem[2 * j] -= __bfloat162float(t.x);
                    rem[2 * j + 1] -= __bfloat162float(t.y);
                }
                float o2[8];
                mma_h16(o2, r[0], r[1], r[2], r[3], hf);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] += o2[e];
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) v[h][e] = o[e];
    }
    stage_e2(v);
    stage_rows<1>(v);
    stage_rows<2>(v);
    stage_rows<4>(v);
    warp_transpose(v, scratch, lane);
    if (logb >= 9) stage_rows<1>(v);
    if (logb >= 10) stage_rows<2>(v);
    if (logb >= 11) stage_rows<4>(v);
    uint16_t* dq = dq_tile;
    int tc = (wbase + 8 * lane) % C, tr = (wbase + 8 * lane) / C;  // column, row of chunk 0
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int col = tc, rowk = tr;
        tc += 256;
        if (tc >= C) { tc -= C; ++tr; }
        if (k >= nchunks) continue;
        const int te = wbase + 256 * k + 8 * lane;  // tile element of the 8-run
        const float m = rowm[win_rows ? row_w : rowk];
        unsigned o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 t = __floats2bfloat162_rn(v[k][2 * j] * m, v[k][2 * j + 1] * m);
            o[j] = *reinterpret_cast<const unsigned*>(&t);
        }
        apply_signs(o, __ldg(reinterpret_cast<const uint2*>(signs + col)));
        __stcs(reinterpret_cast<uint4*>(dq + te), make_uint4(o[0], o[1], o[2], o[3]));  // written once: streaming
    }
}

template <int MAXM>
__device__ __forceinline__ FastTile make_tile(const EncodeParams<MAXM>& p, int t) {
    FastTile ft;
    ft.t = t;
    ft.ne = ft.no = 0;
    if (t < p.n_tiles) {
        ft.mat = find_matrix(p, t);
        const MatDesc& M = p.m[ft.mat];
        const int rpt = meta_rpt(M.meta);
        ft.r0 = (t - M.tile_base) * rpt;
        ft.nr = min(rpt, M.rows - ft.r0);
    } else {
        ft.mat = 0;
        ft.r0 = 0;
        ft.nr = 0;
    }
    return ft;
}

// Row scales of a tile, from its input: the blockwise RHT is orthonormal,
// so the rotated row's sum of squares is the (sign-flipped) input row's.
// One warp, rows in turn, fixed summation order; a row whose sum is not
// finite is summed again with non-finite inputs read as 0, as the transform
// reads them.  s_r = sqrt(sum / C) / kappa (or the given scale).
template <int MAXM>
__device__ __forceinline__ void tile_scales(const EncodeParams<MAXM>& p, const FastTile& ft, const uint16_t* tb,
                                            float* rows, float* rowc, float* rowm, int lane) {
    const MatDesc& M = p.m[ft.mat];
    const int C = M.cols;
    const float sqb = sqrtf(static_cast<float>(1 << meta_logb(M.meta)));
    for (int r = 0; r < ft.nr; ++r) {
        const uint4* row = reinterpret_cast<const uint4*>(tb + r * C);
        float ss = 0.f;
        if (!p.scale_in) {
            float2 acc = make_float2(0.f, 0.f);
            for (int k = lane; k < C / 8; k += 32) {
                const uint4 v = row[k];
                const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 t = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
                    acc = __ffma2_rn(t, t, acc);
                }
            }
            ss = acc.x + acc.y;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
            ss = __shfl_sync(0xFFFFFFFFu, ss, 0);
            if (!isfinite(ss)) {
                acc = make_float2(0.f, 0.f);
                for (int k = lane; k < C / 8; k += 32) {
                    const uint4 v = row[k];
                    const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        unsigned x = w[j];
                        if ((x & 0x7F80u) == 0x7F80u) x &= 0xFFFF0000u;
                        if ((x & 0x7F800000u) == 0x7F800000u) x &= 0x0000FFFFu;
                        const float2 t = make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
                        acc = __ffma2_rn(t, t, acc);
                    }
                }
                ss = acc.x + acc.y;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
                ss = __shfl_sync(0xFFFFFFFFu, ss, 0);
            }
        }
        if (lane == 0) {
            float sc;
            if (p.scale_in) {
                sc = M.scale[ft.r0 + r];
                if (!(sc > 0.f) || !isfinite(sc)) sc = 0.f;
            } else {
                sc = sqrtf(ss / static_cast<float>(C)) / p.kappa;
                M.scale[ft.r0 + r] = sc;
            }
            rows[r] = sc;
            rowc[r] = sc > 0.f ? 2.0f / (sc * sqb) : 0.f;
            rowm[r] = sc / sqb;
        }
    }
}

// kSG: the shape-gain code instead of the lattice projection (a separate
// instantiation, so that the projection's code is the same with or without it).
template <int MAXM, bool kSG = false>
__global__ void __launch_bounds__(kFastThreads, 1) k_encode_fast(const __grid_constant__ EncodeParams<MAXM> p,
                                                                  int16_t* __restrict__ ovf_scratch_all) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t* inbuf = reinterpret_cast<uint16_t*>(smem + kFsIn);
    uint16_t* st2 = reinterpret_cast<uint16_t*>(smem + kFsT2);
    uint32_t* smap = reinterpret_cast<uint32_t*>(smem + kFsMap);
    uint32_t* schunk = reinterpret_cast<uint32_t*>(smem + kFsChunk);

    __shared__ __align__(8) uint64_t s_full[2];
    __shared__ FastTile s_info[8];  // tile of iteration i at i & 7
    __shared__ float s_rows[2][kMaxTileRows], s_rowc[2][kMaxTileRows], s_rowm[2][kMaxTileRows];
    __shared__ unsigned s_tot[kFastSlots][2];  // a tile's escape / overflow record counts
    __shared__ unsigned s_ex[kFastSlots][2];   // records of all earlier tiles

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool service = warp == kFastWarps;
    int16_t* ovf_scratch = ovf_scratch_all + static_cast<size_t>(blockIdx.x) * kFastSlots * kFastTileGroups * 8;
    unsigned long long* status = p.ws + 2;

    for (int i = tid; i < 2 * 2401; i += kFastThreads) st2[i] = g_t2[i];  // rank table T2
    if (tid == 0) {
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        fence_mbar_init();
        for (int s = 0; s < 8; ++s) s_info[s] = make_tile(p, 0x7FFFFFFF);
        const int t0 = static_cast<int>(atomicAdd(&p.ws[0], 1ull));
        s_info[0] = make_tile(p, t0);
        if (t0 < p.n_tiles) {
            const FastTile& ft = s_info[0];
            const MatDesc& M = p.m[ft.mat];
            const unsigned bytes = static_cast<unsigned>(ft.nr) * M.cols * 2u;
            mbar_arrive_expect_tx(&s_full[0], bytes);
            bulk_load_hint(inbuf, static_cast<const uint16_t*>(M.w) + static_cast<size_t>(ft.r0) * M.cols, bytes,
                           &s_full[0], l2_policy_evict_first());
        }
    }
    __syncthreads();
    if (service && s_info[0].t < p.n_tiles) {  // row scales of the first tile
        int spins = 0;
        while (!mbar_try_wait(&s_full[0], 0)) {
            if (++spins > kWaitLimit) {
                if (lane == 0) atomicOr(&p.ctr->err, 2ull);
                break;
            }
        }
        tile_scales(p, s_info[0], inbuf, s_rows[0], s_rowc[0], s_rowm[0], lane);
    }
    __syncthreads();

    const HFrag hf = make_hfrag(lane);
    unsigned nonfinite = 0, clamped = 0;  // per thread: at most 64 a tile

    // Iteration i: compute warps transform, project and count tile i and emit
    // the records of tile i - 3; the service warp claims and loads tile i + 1,
    // publishes tile i - 1's record counts and stores its indices, places
    // tile i - 2 among all earlier tiles, and computes tile i + 1's row
    // scales.  One barrier per iteration.
    for (int i = 0;; ++i) {
        // tile descriptors stay in shared memory (the service warp writes only slot i + 1)
        const FastTile& cur = s_info[i & 7];
        const FastTile& prev1 = s_info[(i + 7) & 7];
        const FastTile& prev2 = s_info[(i + 6) & 7];
        const FastTile& prev3 = s_info[(i + 5) & 7];
        const bool cur_ok = cur.t < p.n_tiles, p1_ok = i >= 1 && prev1.t < p.n_tiles,
                   p2_ok = i >= 2 && prev2.t < p.n_tiles, p3_ok = i >= 3 && prev3.t < p.n_tiles;
        if (!cur_ok && !p1_ok && !p2_ok && !p3_ok) break;
        const int b = i & 1, sl = i & 3, sl1 = (i + 3) & 3, sl2 = (i + 2) & 3, sl3 = (i + 1) & 3;

        if (!service) {
            // ================================================ compute warps
            if (cur_ok) {
                const MatDesc& M = p.m[cur.mat];
                const int C = M.cols, gpr = C >> 3, logb = meta_logb(M.meta);
                const int n = cur.nr * C, G = cur.nr * gpr;
                const int nwin = (n + 2047) >> 11;
                const bool win_rows = (C & 2047) == 0;  // every window inside one row
                const float* rows_b = s_rows[b];
                const float* rowc_b = s_rowc[b];
                const float* rowm_b = s_rowm[b];
                float v[8][8];
                const int w = warp;
                const int wbase = 2048 * w;
                const int nchunks = max(0, min(8, (n - wbase) >> 8));
                uint16_t* win = inbuf + b * kFastTileElems + wbase;
                float4* scratch = reinterpret_cast<float4*>(win);
                if (w < nwin) {
                    {  // wait for the tile's bytes (bounded)
                        int spins = 0;
                        while (!mbar_try_wait(&s_full[b], (i >> 1) & 1)) {
                            if (++spins > kWaitLimit) {
                                if (lane == 0) atomicOr(&p.ctr->err, 2ull);
                                break;
                            }
                        }
                    }
                    // a window with a non-finite input runs again from a copy of its
                    // input in which those values read as 0 (one copy of the transform)
#pragma unroll 1
                    for (int pass = 0; pass < 2; ++pass) {
                        if (pass == 1) {
                            sanitize_window(win, static_cast<const uint16_t*>(M.w) + static_cast<size_t>(cur.r0) * C + wbase,
                                            nchunks, lane, nonfinite);
                            __syncwarp();
                        }
                        unsigned raw[8][4];
                        load_window_raw(raw, win, false, M.signs, C, wbase, nchunks, lane, nonfinite);
                        __syncwarp();
                        const float ss = window_forward(v, raw, logb, nchunks, scratch, lane, hf);
                        if (!__any_sync(0xFFFFFFFFu, !isfinite(ss))) break;
                    }
                }
                // projection + encoding of the warp's 8 x 32 groups
                uint32_t* map = smap + sl * kFastTileGroups;
                uint16_t* idxs = M.idx + static_cast<size_t>(cur.r0) * gpr;
                int16_t* oscr = ovf_scratch + static_cast<size_t>(sl) * kFastTileGroups * 8;
                if (w < nwin) {
                    const int a = lane >> 2, q = lane & 3;
                    const bool lane_ok = a < nchunks;
                    const int row_w = win_rows ? (wbase / C) : 0;
                    // row of the lane's groups: its 8 groups span 232 elements, so the row
                    // advances at most once (at hcut) when the width is not a multiple of 2048
                    const int e0 = 8 * (256 * w + 32 * a + q);
                    const int r0l = e0 / C, hcut = (C - e0 % C + 31) >> 5;
                    bool big = false;  // some |P_i| > 255 (|P|^2 > 65025), or a shape-gain reconstruction
                    if (kSG) {
                        // shape-gain code (sg_code): the 16-bit code is the map word (no
                        // record), the reconstruction x-hat = xm P, held doubled in v for the dequant
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const int row = win_rows ? row_w : r0l + (h >= hcut ? 1 : 0);
                            const float c = rowc_b[lane_ok ? row : 0];
                            float X[8];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 t = __fmul2_rn(make_float2(v[h][2 * j], v[h][2 * j + 1]), make_float2(c, c));
                                X[2 * j] = t.x;
                                X[2 * j + 1] = t.y;
                            }
                            if (p.clamp) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) X[e] = fminf(fmaxf(X[e], -1048576.f), 1048576.f);
                            }
                            int Pi[8];
                            float xm;
                            const int code = sg_code(X, Pi, xm, g_t1, st2);
#pragma unroll
                            for (int e = 0; e < 8; ++e) v[h][e] = 2.f * xm * static_cast<float>(Pi[e]);
                            if (lane_ok) map[map_slot(256 * w + 32 * a + 4 * h + q)] = static_cast<uint32_t>(code);
                        }
                        big = true;  // x-hat has up to 9 significant bits: the three-term bf16 split
                        __syncwarp();
                    } else {
                        // the lane's 8 groups are independent: project all of them, then
                        // rank all of them, then queue, so that the chains overlap
                        unsigned oddm = 0u;
    #pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const int row = win_rows ? row_w : r0l + (h >= hcut ? 1 : 0);
                            const float c = rowc_b[lane_ok ? row : 0];
                            float X[8];
    #pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 t = __fmul2_rn(make_float2(v[h][2 * j], v[h][2 * j + 1]), make_float2(c, c));
                                X[2 * j] = t.x;
                                X[2 * j + 1] = t.y;
                            }
                            if (p.clamp) {
    #pragma unroll
                                for (int e = 0; e < 8; ++e) X[e] = fminf(fmaxf(X[e], -1048576.f), 1048576.f);
                            }
                            float Pf[8];
                            oddm |= (e8_nearest_lean(X, Pf) ? 1u : 0u) << h;
    #pragma unroll
                            for (int e = 0; e < 8; ++e) v[h][e] = Pf[e];  // keep p for the dequant
                        }
                        // Groups that may lie outside the core: the core holds every point with
                        // |p|^2 <= 10 and none with |p|^2 > 12, so only |P|^2 > 40 can escape.
                        // Their extended rank comes straight from the coordinates (digits
                        // (P + 9) >> 1 = P / 2 + 4 or + 4.5, keys base 10, exact in fp32); the two
                        // table gathers of all 8 groups are issued together with the core ranks,
                        // so that their latency overlaps them, and the encoding words after them.
                        // These tables are read through L2 only (__ldcg): their scattered
                        // lines would otherwise push the rank table T1 out of L1.
                        uint32_t ia[8], ib[8];
                        int rks[8];
    #pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const float (&P)[8] = v[h];
                            float2 n = __fmul2_rn(make_float2(P[0], P[4]), make_float2(P[0], P[4]));
                            n = __ffma2_rn(make_float2(P[1], P[5]), make_float2(P[1], P[5]), n);
                            n = __ffma2_rn(make_float2(P[2], P[6]), make_float2(P[2], P[6]), n);
                            n = __ffma2_rn(make_float2(P[3], P[7]), make_float2(P[3], P[7]), n);
                            const float n2 = n.x + n.y;
                            big |= !(n2 <= 65025.f);
                            const bool in = lane_ok && n2 > 40.f && n2 <= 88.f;  // then every |P_i| <= 9 as well
                            float2 k = __fmul2_rn(make_float2(P[0], P[4]), make_float2(1000.f, 1000.f));
                            k = __ffma2_rn(make_float2(P[1], P[5]), make_float2(100.f, 100.f), k);
                            k = __ffma2_rn(make_float2(P[2], P[6]), make_float2(10.f, 10.f), k);
                            k = __fadd2_rn(make_float2(P[3], P[7]), k);
                            const float base = ((oddm >> h) & 1u) ? 14999.5f : 4444.f;  // type * 10000 + 1111 * (4.5 or 4)
                            const int hk = __float_as_int(fmaf(k.x, 0.5f, base) + 8388608.f) - 0x4B000000;
                            const int lk = __float_as_int(fmaf(k.y, 0.5f, base) + 8388608.f) - 0x4B000000;
                            const int lv = __float_as_int(fmaf(n2, 0.125f, 8388608.f)) - 0x4B000000;
                            ia[h] = in ? __ldcg(g_t1e + hk * 12 + lv) : 0xFFFFFFFFu;
                            ib[h] = in ? __ldcg(g_t2e + lk) : 0xFFFFFFFFu;
                            rks[h] = lane_ok ? core_rank_nb(P, (oddm >> h) & 1u, n2, g_t1, st2) : 0;
                        }
                        uint32_t ew[8];
                        unsigned pendm = 0u;
    #pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const bool pend = lane_ok && rks[h] < 0;
                            pendm |= (pend ? 1u : 0u) << h;
                            const uint32_t r = ia[h] + ib[h];
                            const bool hit = pend && ia[h] != 0xFFFFFFFFu && ib[h] != 0xFFFFFFFFu &&
                                             r < static_cast<uint32_t>(kExtPoints);
                            ew[h] = hit ? __ldcg(g_res + r) : (2u << 24);
                        }
    #pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            if (!lane_ok) continue;
                            const int gt = 256 * w + 32 * a + 4 * h + q;
                            const bool pend = (pendm >> h) & 1u;
                            const uint32_t word = pend ? ew[h] : static_cast<uint32_t>(rks[h]);
                            map[map_slot(gt)] = word;
                            // an overflow record keeps the coordinates as int16 (saturated when
                            // the inputs were clamped); formed for every group, without a branch:
                            // x + 1.5 * 2^23 holds the integer x in its low 16 bits (|x| < 2^22)
                            const bool ovf = pend && (word >> 24) == 2;
                            float c[8];
                            bool clamp = false;
    #pragma unroll
                            for (int k = 0; k < 8; ++k) c[k] = v[h][k];
                            if (p.clamp) {
    #pragma unroll
                                for (int k = 0; k < 8; ++k) {
                                    const float t = fminf(fmaxf(c[k], -32768.f), 32767.f);
                                    clamp |= t != c[k];
                                    c[k] = t;
                                }
                            }
                            unsigned o[4];
    #pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 t = __fadd2_rn(make_float2(c[2 * j], c[2 * j + 1]), make_float2(12582912.f, 12582912.f));
                                o[j] = prmt(__float_as_uint(t.x), __float_as_uint(t.y), 0x5410u);
                            }
                            if (ovf) *reinterpret_cast<uint4*>(oscr + 8 * gt) = make_uint4(o[0], o[1], o[2], o[3]);
                            if (ovf && clamp) ++clamped;
                        }
                        __syncwarp();
                    }
                    // dequantised weights
                    if (p.dq_mode == E8Q_DEQUANT_ROTATED) {
                        uint16_t* dq = static_cast<uint16_t*>(M.dq) + static_cast<size_t>(cur.r0) * C;
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            if (!lane_ok) continue;
                            const int gt = 256 * w + 32 * a + 4 * h + q;
                            const float s = rows_b[win_rows ? row_w : r0l + (h >= hcut ? 1 : 0)];
                            uint4 o;
                            o.x = bf16x2_of_half_products(s, v[h][0], v[h][1]);
                            o.y = bf16x2_of_half_products(s, v[h][2], v[h][3]);
                            o.z = bf16x2_of_half_products(s, v[h][4], v[h][5]);
                            o.w = bf16x2_of_half_products(s, v[h][6], v[h][7]);
                            __stcs(reinterpret_cast<uint4*>(dq + 8 * gt), o);
                        }
                    } else if (p.dq_mode == E8Q_DEQUANT_ORIGINAL) {
                        window_dequant_original(v, scratch, lane, hf, logb,
                                                static_cast<uint16_t*>(M.dq) + static_cast<size_t>(cur.r0) * C, M.signs, C,
                                                wbase, nchunks, rowm_b, win_rows, row_w, big ? 1 : 0);
                    }
                }
                if (w < nwin) {
                    // the window's record counts per 32-group chunk and its indices;
                    // its records are compacted, in group order, over its own 256 map
                    // entries: local group << 24 | root << 16 | core index, the root
                    // field 0xFF for an overflow record.  A record lands at or before
                    // the slots of its own chunk, all read before the chunk's ballots.
                    uint32_t* cnt = schunk + sl * 2 * kFastCnt;
                    uint32_t* wl = map + 256 * w;
                    unsigned run = 0;
                    const unsigned lt = lanemask_lt();
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int c = 8 * w + k;
                        if (32 * c >= G) break;
                        const int g = 32 * c + lane;
                        const uint32_t m = g < G ? map[map_slot(g)] : 0u;
                        const uint32_t kind = m >> 24;
                        if (g < G) __stcs(idxs + g, static_cast<unsigned short>(kind == 2 ? 0u : (m & 0xFFFFu)));
                        const unsigned be = __ballot_sync(0xFFFFFFFFu, kind == 1), bo = __ballot_sync(0xFFFFFFFFu, kind == 2);
                        if (lane == 0) {
                            cnt[c] = __popc(be);
                            cnt[kFastCnt + c] = __popc(bo);
                        }
                        if (kind != 0)
                            wl[run + __popc((be | bo) & lt)] =
                                (static_cast<uint32_t>(32 * k + lane) << 24) | (kind == 1 ? (m & 0xFFFFFFu) : 0xFF0000u);
                        run += __popc(be | bo);
                    }
                }
            }
            // emit the records of tile i - 3, placed by the service warp during
            // the previous iteration: each warp copies its own window's compacted
            // list, escape and overflow records each to their contiguous range
            if (p3_ok) {
                const MatDesc& M = p.m[prev3.mat];
                const int gpr = M.cols >> 3, G = prev3.nr * gpr, nch = (G + 31) >> 5;
                const uint32_t* cnt = schunk + sl3 * 2 * kFastCnt;
                const long long ex_e = s_ex[sl3][0], ex_o = s_ex[sl3][1];
                if (8 * warp < nch) {
                    const int c0 = 8 * warp;
                    const uint32_t* wl = smap + sl3 * kFastTileGroups + 256 * warp;
                    const int16_t* oscr = ovf_scratch + (static_cast<size_t>(sl3) * kFastTileGroups + 256 * warp) * 8;
                    const uint32_t gw = M.group_base + static_cast<uint32_t>(prev3.r0) * gpr + 256u * warp;
                    long long pe = ex_e + cnt[c0], po = ex_o + cnt[kFastCnt + c0];
                    // (at most the window's 256 groups: the bound keeps every list read
                    // inside the window's part of the map)
                    const int n = min(256, static_cast<int>((cnt[c0 + 8] - cnt[c0]) +
                                                            (cnt[kFastCnt + c0 + 8] - cnt[kFastCnt + c0])));
                    const unsigned lt = lanemask_lt();
                    for (int j0 = 0; j0 < n; j0 += 32) {
                        const int j = j0 + lane;
                        const uint32_t e = j < n ? wl[j] : 0u;
                        const bool ov = j < n && ((e >> 16) & 0xFFu) == 0xFFu;
                        const bool es = j < n && !ov;
                        const unsigned be = __ballot_sync(0xFFFFFFFFu, es), bo = __ballot_sync(0xFFFFFFFFu, ov);
                        const uint32_t lg = e >> 24;
                        if (es) {
                            const long long pos = pe + __popc(be & lt);
                            if (pos < p.esc_cap) __stcs(reinterpret_cast<uint2*>(p.esc + pos), make_uint2(gw + lg, e & 0xFFFFFFu));
                        } else if (ov) {
                            const long long pos = po + __popc(bo & lt);
                            if (pos < p.ovf_cap) {
                                const uint4 cw = *reinterpret_cast<const uint4*>(oscr + 8 * lg);
                                uint32_t* dst = reinterpret_cast<uint32_t*>(p.ovf + pos);
                                dst[0] = gw + lg;
                                dst[1] = cw.x; dst[2] = cw.y; dst[3] = cw.z; dst[4] = cw.w;
                            }
                        }
                        pe += __popc(be);
                        po += __popc(bo);
                    }
                }
                for (int r = tid; r < prev3.nr; r += kFastWarps * 32) {
                    const int c = (r * gpr) >> 5;  // rows start on chunk boundaries (gpr % 32 == 0)
                    if (p.esc_rp) p.esc_rp[M.row_base + prev3.r0 + r] = ex_e + cnt[c];
                    if (p.ovf_rp) p.ovf_rp[M.row_base + prev3.r0 + r] = ex_o + cnt[kFastCnt + c];
                }
                if (prev3.t == p.n_tiles - 1 && tid == 0) {
                    const long long te = ex_e + cnt[kFastChunks], to = ex_o + cnt[kFastCnt + kFastChunks];
                    if (p.esc_rp) p.esc_rp[p.total_rows] = te;
                    if (p.ovf_rp) p.ovf_rp[p.total_rows] = to;
                    p.ctr->n_escape = te;
                    p.ctr->n_overflow = to;
                    p.ctr->n_dropped = (te > p.esc_cap ? te - p.esc_cap : 0) + (to > p.ovf_cap ? to - p.ovf_cap : 0);
                }
            }
            fence_proxy_async_smem();
        } else if (service) {
            // ================================================= service warp
            if (lane == 0) {
                int tn = 0x7FFFFFFF;
                if (cur_ok) tn = static_cast<int>(atomicAdd(&p.ws[0], 1ull));
                const FastTile nt = make_tile(p, tn);
                s_info[(i + 1) & 7] = nt;
                if (tn < p.n_tiles) {
                    const MatDesc& M = p.m[nt.mat];
                    const unsigned bytes = static_cast<unsigned>(nt.nr) * M.cols * 2u;
                    uint64_t* bar = &s_full[(i + 1) & 1];
                    mbar_arrive_expect_tx(bar, bytes);
                    // the latent weights are read once: their L2 lines go first, so that
                    // the lookup tables stay in L2
                    bulk_load_hint(inbuf + ((i + 1) & 1) * kFastTileElems,
                                   static_cast<const uint16_t*>(M.w) + static_cast<size_t>(nt.r0) * M.cols, bytes, bar,
                                   l2_policy_evict_first());
                }
            }
            __syncwarp();
            if (p1_ok) {  // tile i - 1: chunk prefix (group order), publish its counts
                const MatDesc& M = p.m[prev1.mat];
                const int gpr = M.cols >> 3, nch = (prev1.nr * gpr + 31) >> 5;
                uint32_t* cnt = schunk + sl1 * 2 * kFastCnt;
                constexpr int kPer = (kFastChunks + 31) / 32;  // chunks per lane: lane + 32 k
                unsigned ne = 0, no = 0;  // running totals of the earlier rounds
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    const int c = lane + 32 * k;
                    const unsigned ce = c < nch ? cnt[c] : 0u, co = c < nch ? cnt[kFastCnt + c] : 0u;
                    unsigned se = ce, so = co;  // inclusive scans
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const unsigned a0 = __shfl_up_sync(0xFFFFFFFFu, se, off), b0 = __shfl_up_sync(0xFFFFFFFFu, so, off);
                        if (lane >= off) { se += a0; so += b0; }
                    }
                    if (c < kFastChunks) {
                        cnt[c] = ne + se - ce;
                        cnt[kFastCnt + c] = no + so - co;
                    }
                    ne += __shfl_sync(0xFFFFFFFFu, se, 31);
                    no += __shfl_sync(0xFFFFFFFFu, so, 31);
                }
                if (lane == 0) {
                    cnt[kFastChunks] = ne;
                    cnt[kFastCnt + kFastChunks] = no;
                    s_tot[sl1][0] = ne;
                    s_tot[sl1][1] = no;
                    const unsigned long long own = (static_cast<unsigned long long>(ne) << 31) | no;
                    st_volatile_u64(&status[prev1.t], (prev1.t == 0 ? (2ull << 62) : (1ull << 62)) | own);
                }
            }
            __syncwarp();
            if (p2_ok) {  // tile i - 2: its place among all earlier tiles' records
                unsigned ex_e = 0, ex_o = 0;
                if (prev2.t > 0) {
                    unsigned acc_e = 0, acc_o = 0;
                    int j = prev2.t - 1, spins = 0;
                    while (true) {
                        const int k = j - lane;
                        const unsigned long long st = (k >= 0) ? ld_volatile_u64(&status[k]) : (2ull << 62);
                        const unsigned flag = static_cast<unsigned>(st >> 62);
                        const unsigned notready = __ballot_sync(0xFFFFFFFFu, flag == 0);
                        const unsigned ispre = __ballot_sync(0xFFFFFFFFu, flag == 2);
                        const unsigned window = ispre ? (((ispre & (0u - ispre)) << 1) - 1u) : 0xFFFFFFFFu;
                        if (notready & window) {
                            if (++spins > kSpinLimit) {
                                if (lane == 0) atomicOr(&p.ctr->err, 1ull);
                                break;
                            }
                            __nanosleep(64);
                            continue;
                        }
                        const bool in = (window >> lane) & 1u;
                        unsigned ve = in ? static_cast<unsigned>((st >> 31) & 0x7FFFFFFFu) : 0u;
                        unsigned vo = in ? static_cast<unsigned>(st & 0x7FFFFFFFu) : 0u;
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
                    ex_e = acc_e;
                    ex_o = acc_o;
                    if (lane == 0)
                        st_volatile_u64(&status[prev2.t],
                                        (2ull << 62) |
                                            (static_cast<unsigned long long>((ex_e + s_tot[sl2][0]) & 0x7FFFFFFFu) << 31) |
                                            ((ex_o + s_tot[sl2][1]) & 0x7FFFFFFFu));
                }
                if (lane == 0) {
                    s_ex[sl2][0] = ex_e;
                    s_ex[sl2][1] = ex_o;
                }
            }
            {  // row scales of tile i + 1 once its bytes are in
                const FastTile nt = s_info[(i + 1) & 7];
                if (nt.t < p.n_tiles) {
                    int spins = 0;
                    while (!mbar_try_wait(&s_full[(i + 1) & 1], ((i + 1) >> 1) & 1)) {
                        if (++spins > kWaitLimit) {
                            if (lane == 0) atomicOr(&p.ctr->err, 2ull);
                            break;
                        }
                    }
                    tile_scales(p, nt, inbuf + ((i + 1) & 1) * kFastTileElems, s_rows[(i + 1) & 1],
                                s_rowc[(i + 1) & 1], s_rowm[(i + 1) & 1], lane);
                }
            }
            __syncwarp();
        }
        __syncthreads();
    }

    unsigned long long nf = nonfinite, cl = clamped;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        nf += __shfl_xor_sync(0xFFFFFFFFu, nf, off);
        cl += __shfl_xor_sync(0xFFFFFFFFu, cl, off);
    }
    if (lane == 0) {
        if (nf) atomicAdd(&p.ctr->n_nonfinite, nf);
        if (cl) atomicAdd(&p.ctr->n_clamped, cl);
    }
}

}  // namespace e8q
