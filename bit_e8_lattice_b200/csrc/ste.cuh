// Identity straight-through estimator, backward ("E8-QAT", Figure 2 (b):
// projection with an identity STE): the latents' gradient is the gradient
// of the dequantised weights, element for element.  When the caller gives
// two buffers the gradient is copied; an aliased call launches nothing.
#pragma once
#include <cstdint>

namespace e8q {

constexpr int kSteThreads = 512;
constexpr int kSteUnroll = 4;  // 16-byte words in flight per thread

// n16: 16-byte words (both pointers 16-byte aligned); grid-stride, the
// loads of a round issued before its stores.
__global__ void __launch_bounds__(kSteThreads) k_ste_copy16(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                            long long n16) {
    const long long stride = static_cast<long long>(gridDim.x) * kSteThreads;
    long long i = static_cast<long long>(blockIdx.x) * kSteThreads + threadIdx.x;
    for (; i + (kSteUnroll - 1) * stride < n16; i += kSteUnroll * stride) {
        uint4 v[kSteUnroll];
#pragma unroll
        for (int u = 0; u < kSteUnroll; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kSteUnroll; ++u) __stcs(dst + i + u * stride, v[u]);
    }
    for (; i < n16; i += stride) __stcs(dst + i, __ldcs(src + i));
}

// Element copy for buffers that are not both 16-byte aligned, and for the
// tail of the aligned copy.
__global__ void __launch_bounds__(kSteThreads) k_ste_copy2(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst,
                                                           long long n) {
    const long long stride = static_cast<long long>(gridDim.x) * kSteThreads;
    for (long long i = static_cast<long long>(blockIdx.x) * kSteThreads + threadIdx.x; i < n; i += stride)
        dst[i] = src[i];
}

}  // namespace e8q
