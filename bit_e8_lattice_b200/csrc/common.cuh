// Shared device helpers: constant tables, launch descriptors, small
// Hadamard butterflies.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/e8q.h"

namespace e8q {

constexpr int kMaxMats = 448;
constexpr int kTileMaxElems = 16384;  // elements of one row tile (fp32 in shared memory)
constexpr int kTileMaxGroups = kTileMaxElems / 8;
constexpr int kMaxTileRows = 64;
constexpr int kMaxCols = 16384;

// Constant tables, one copy per device, filled once from the host.
__device__ __align__(16) uint16_t g_t1[2 * 2401 * 7];
__device__ __align__(16) uint16_t g_t2[2 * 2401];
__device__ __align__(16) uint2 g_core8[65536];  // 8 int8 doubled coordinates per core index
__device__ __align__(16) uint2 g_root8[240];
__device__ __align__(16) uint8_t g_rootkey[512];  // root index by construction key
// Escape lookup over every E8 point with |P|^2 <= 88 (host tables.h): the
// two-table extended rank and the encoding word of each extended point.
constexpr int kExtPoints = 1113841;
__device__ __align__(16) uint32_t g_t1e[2 * 10000 * 12];
__device__ __align__(16) uint32_t g_t2e[2 * 10000];
__device__ __align__(16) uint32_t g_res[kExtPoints];

// Rows per tile: enough rows that a tile holds about 4K elements.
__host__ __device__ inline int rows_per_tile(int cols) {
    int r = 4096 / cols;
    return r < 1 ? 1 : (r > kMaxTileRows ? kMaxTileRows : r);
}

struct MatDesc {  // 64 bytes
    const void* w;
    const int8_t* signs;
    uint16_t* idx;
    float* scale;
    void* dq;
    int32_t rows;
    int32_t cols;
    int32_t meta;       // bits 0..3 log2(B) (0: no transform); bit 4 bf16 input; bits 8..15 rows per tile
    int32_t tile_base;  // first tile id of this matrix
    int32_t row_base;   // first CSR row of this matrix
    uint32_t group_base;
};
static_assert(sizeof(MatDesc) == 64, "descriptor layout");

__device__ __forceinline__ int meta_logb(int meta) { return meta & 0xF; }
__device__ __forceinline__ bool meta_bf16(int meta) { return (meta >> 4) & 1; }
__device__ __forceinline__ int meta_rpt(int meta) { return (meta >> 8) & 0xFF; }

// In-register Sylvester butterflies on m = 2, 4 or 8 values.
template <int M>
__device__ __forceinline__ void fwht_reg(float (&v)[8]) {
#pragma unroll
    for (int h = 1; h < M; h <<= 1)
#pragma unroll
        for (int i = 0; i < M; ++i)
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

// Unnormalised blockwise Hadamard transform of n floats in shared memory
// (blocks of 2^logb), radix-8 passes, whole CTA; ends with a barrier.
__device__ inline void fwht_smem(float* buf, int n, int logb) {
    for (int s = 0; s < logb; s += 3) {
        const int k = (logb - s) < 3 ? (logb - s) : 3;
        const int h = 1 << s, m = 1 << k;
        const int nsets = n >> k;
        for (int q = threadIdx.x; q < nsets; q += blockDim.x) {
            const int lo = q & (h - 1);
            const int base = ((q >> s) << (s + k)) | lo;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < m) v[j] = buf[base + j * h];
            if (k == 3) fwht_reg<8>(v);
            else if (k == 2) fwht_reg<4>(v);
            else fwht_reg<2>(v);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < m) buf[base + j * h] = v[j];
        }
        __syncthreads();
    }
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ unsigned long long ld_volatile_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_volatile_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

}  // namespace e8q
