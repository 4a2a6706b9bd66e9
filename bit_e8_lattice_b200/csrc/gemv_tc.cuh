// K5 on the 5th-generation tensor cores ("E8-QAT", abstract: decoding
// throughput of the 2-bit representation):
//
//   D[r][b] = sum_k A[r][k] X[b][k],   A = doubled codeword coordinates P
//   (exact in fp16; escape roots added, overflow groups zero), X = xr_b * 2^-e_b
//   in fp16 (the prep kernel's scaling), D in fp32 in tensor memory.
//
// Work units are (128-row tile, contiguous range of 64-column K tiles); the
// K range of a row tile is split so that there are about two units per SM,
// and persistent CTAs take units round-robin.  Each unit's fp32 partial sums
// go to the workspace; k_gv_fin adds the splits in a fixed order, scales them
// and applies the overflow records.
//
// Warp roles in a CTA (21 warps):
// - 16 producer warps fill a ring of 4 shared-memory stages.  Per K tile a
//   thread decodes 2 groups of one row (indices loaded four tiles ahead,
//   codeword words from a shared-memory copy of the table's first entries,
//   else through L1; root bytes added; nibbles -> fp16 pairs) into the A
//   stage, and asynchronous copies bring the activations into the B stage,
//   both in the K-major core-matrix layout without swizzle (8 rows x 16 bytes
//   per core matrix, next 8 columns 128 bytes on, next 8 rows 1 KB on).  The
//   thread then fences its writes for the tensor cores and arrives on the
//   stage's "full" mbarrier.
// - 1 MMA warp: one thread waits for a full stage, issues its 4 MMAs of
//   K = 16 (M = 128, N = the batch rounded up to 16) into one of two
//   tensor-memory accumulators and commits them to the stage's "empty"
//   mbarrier; after a unit's last stage it commits to the accumulator's
//   "full" mbarrier.
// - 4 epilogue warps (one per 32-lane quarter of tensor memory) read a
//   finished accumulator with tcgen05.ld, store the unit's partial sums and
//   release the accumulator, so that the next unit's MMAs overlap them.
// Every wait is bounded; a wait that gives up sets a device error flag.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemv.cuh"
#include "ptx.cuh"

namespace e8q {

constexpr int kTcRows = 128;   // M: weight rows per tile (tensor-memory lanes)
constexpr int kTcKCols = 64;   // K columns per stage: 8 groups, 4 MMAs of K = 16
constexpr int kTcStages = 4;
constexpr int kTcProdWarps = 16;
constexpr int kTcMmaWarp = kTcProdWarps;                // warp 16; the epilogue warps are 17..20
constexpr int kTcThreads = (kTcProdWarps + 1 + 4) * 32;
constexpr int kTcWaitLimit = 1 << 22;
// batch from which e8q_dequant_gemv picks this kernel by itself: none yet (it
// measures slower than the mma.sync kernel at every batch; e8q_set_gemv_path
// selects it)
constexpr int kTcMinBatch = 1 << 30;
constexpr size_t kTcABytes = size_t{kTcRows} * kTcKCols * 2;  // 16 KB
constexpr size_t kTcSmemCap = 226 * 1024;                      // dynamic shared memory per CTA

__host__ __device__ constexpr size_t tc_b_bytes(int n) { return static_cast<size_t>(n) * kTcKCols * 2; }
__host__ __device__ constexpr size_t tc_stage_bytes(int n) { return kTcABytes + tc_b_bytes(n); }
__host__ __device__ constexpr int tc_tab_fit(int n) {
    return static_cast<int>((kTcSmemCap - kTcStages * tc_stage_bytes(n) - 256 * 8) / 4 / 1024 * 1024);
}
// codeword words held in shared memory: what the stages leave, in units of 1024
__host__ __device__ constexpr int tc_tab_words(int n) { return tc_tab_fit(n) > 65536 ? 65536 : tc_tab_fit(n); }
__host__ __device__ constexpr size_t tc_smem_bytes(int n) {
    return kTcStages * tc_stage_bytes(n) + 256 * 8 + static_cast<size_t>(tc_tab_words(n)) * 4;
}

// bit 0: a bounded wait of the tensor-core GEMV gave up (read by e8q_device_error_flags)
__device__ unsigned long long g_tc_err;

struct GvTcParams {
    const uint16_t* idx;
    const uint8_t* map;  // root map [rows][mstride] (root + 1, 0: none); null: no escapes
    const uint16_t* xk;  // fp16 [batch][cols]: xr * 2^-e
    float* part;         // [nsplit][rows][batch]
    int32_t rows, cols, gpr, batch, mstride;
    int32_t nrt;     // 128-row tiles
    int32_t nkt;     // 64-column K tiles
    int32_t nsplit;  // K ranges per row tile (<= nkt)
    int32_t vec_idx;
};

// Byte offset of (row, 8-column chunk kc) in a stage operand: core matrices
// of 8 rows x 16 bytes, the 8 chunks of a row group 128 bytes apart, row
// groups 1 KB apart.
__device__ __forceinline__ uint32_t tc_core_off(int row, int kc) {
    return static_cast<uint32_t>(((row >> 3) * 8 + kc) * 128 + (row & 7) * 16);
}

// Shared-memory matrix descriptor for that layout (K-major, no swizzle):
// start >> 4, leading byte offset 128 >> 4, stride byte offset 1024 >> 4,
// descriptor version 1.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: fp32 D, fp16 A and B, both K-major, N, M = 128.
__host__ __device__ constexpr uint32_t tc_idesc(int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kTcRows >> 4) << 24);
}

__device__ __forceinline__ unsigned tc_wait(uint64_t* bar, unsigned parity) {
    for (int spins = 0; spins < kTcWaitLimit; ++spins)
        if (mbar_try_wait(bar, parity)) return 0u;
    return 1u;
}

// unit -> row tile, K tiles [k0, k1)
struct TcUnit {
    int rt, split, k0, k1;
};
__device__ __forceinline__ TcUnit tc_unit(const GvTcParams& p, int u) {
    TcUnit t;
    t.rt = u % p.nrt;
    t.split = u / p.nrt;
    t.k0 = static_cast<int>(static_cast<long long>(t.split) * p.nkt / p.nsplit);
    t.k1 = static_cast<int>(static_cast<long long>(t.split + 1) * p.nkt / p.nsplit);
    return t;
}

template <int N>
__global__ void __launch_bounds__(kTcThreads, 1) k_gv_tc(const __grid_constant__ GvTcParams p) {
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N: a multiple of 16 in 16..256 for M = 128");
    constexpr uint32_t kAcc = N;                          // columns of one accumulator
    constexpr uint32_t kCols = 2 * kAcc < 32 ? 32 : 2 * kAcc;  // two accumulators
    static_assert((kCols & (kCols - 1)) == 0 && kCols <= 512, "tensor-memory columns: a power of two <= 512");
    constexpr int kTab = tc_tab_words(N);
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ __align__(8) uint64_t s_full[kTcStages], s_empty[kTcStages], s_accf[2], s_acce[2];
    __shared__ uint32_t s_taddr;
    unsigned char* stages = smem;
    uint2* s_root = reinterpret_cast<uint2*>(smem + kTcStages * tc_stage_bytes(N));
    uint32_t* s_tab = reinterpret_cast<uint32_t*>(smem + kTcStages * tc_stage_bytes(N) + 256 * 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nunits = p.nrt * p.nsplit;
    pdl_launch_dependents();

    // tables (independent of the prep kernel), barriers, tensor memory
    for (int i = tid; i < 256; i += kTcThreads) s_root[i] = gv_root_entry(i);
    for (int i = tid; i < kTab / 4; i += kTcThreads)
        reinterpret_cast<uint4*>(s_tab)[i] = __ldg(reinterpret_cast<const uint4*>(g_gv_tab) + i);
    if (tid == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&s_full[s], kTcProdWarps * 32);
            mbar_init(&s_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&s_accf[a], 1);
            mbar_init(&s_acce[a], 128);
        }
        fence_mbar_init();
    }
    if (warp == kTcMmaWarp) tmem_alloc(&s_taddr, kCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = s_taddr;
    pdl_wait();  // activations and root map written by the prep kernel

    unsigned err = 0;
    if (warp < kTcProdWarps) {
        // ------------------------------------------------------ producers
        // A software pipeline over the CTA's positions (unit, K tile): at step
        // q the thread looks up the codeword words of position q + 2 (indices
        // loaded two steps before), issues the activation copy of position
        // q + 2, decodes position q and loads the indices of position q + 4.
        // row of the tile and groups gq, gq + 1 of a stage: warp w takes rows
        // 8w .. 8w + 7, and the 8 lanes of each quarter-warp store phase take
        // 8 rows of one column chunk -- one whole 128-byte line, no bank conflict
        const int r_l = 8 * (tid >> 5) + (tid & 7), gq = 2 * ((tid >> 3) & 3);
        struct Pos {
            int u, kt, rt, k1;
        };
        auto first = [&]() {
            Pos x;
            x.u = blockIdx.x;
            const TcUnit U = tc_unit(p, x.u < nunits ? x.u : 0);
            x.kt = U.k0;
            x.rt = U.rt;
            x.k1 = U.k1;
            return x;
        };
        auto next = [&](const Pos& x) {
            Pos y = x;
            if (++y.kt >= x.k1) {
                y.u = x.u + static_cast<int>(gridDim.x);
                const TcUnit U = tc_unit(p, y.u < nunits ? y.u : 0);
                y.kt = U.k0;
                y.rt = U.rt;
                y.k1 = U.k1;
            }
            return y;
        };
        auto load_ix = [&](const Pos& x, uint32_t& iv, uint32_t& mv) {
            iv = 0u;
            mv = 0u;
            if (x.u >= nunits) return;
            const int row = x.rt * kTcRows + r_l;
            const int g0 = x.kt * 8 + gq;
            if (row >= p.rows || g0 >= p.gpr) return;
            const uint16_t* ip = p.idx + static_cast<size_t>(row) * p.gpr + g0;
            if (p.vec_idx && g0 + 2 <= p.gpr)
                iv = __ldg(reinterpret_cast<const unsigned*>(ip));
            else
                iv = static_cast<unsigned>(ip[0]) | (g0 + 1 < p.gpr ? static_cast<unsigned>(ip[1]) << 16 : 0u);
            if (p.map) mv = __ldg(reinterpret_cast<const unsigned short*>(p.map + static_cast<size_t>(row) * p.mstride + g0));
        };
        auto words = [&](uint32_t iv, uint32_t (&w)[2]) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const unsigned id = j ? (iv >> 16) : (iv & 0xFFFFu);
                w[j] = id < static_cast<unsigned>(kTab) ? s_tab[id] : __ldg(g_gv_tab + id);
            }
        };
        // activation copy of position x into its stage (after the stage's previous MMAs)
        auto issue_b = [&](const Pos& x, int q) {
            if (x.u < nunits) {
                const int s = q % kTcStages;
                if (q >= kTcStages) err |= tc_wait(&s_empty[s], (static_cast<unsigned>(q / kTcStages) & 1u) ^ 1u);
                unsigned char* bs = stages + s * tc_stage_bytes(N) + kTcABytes;
                for (int c = tid; c < N * 8; c += kTcProdWarps * 32) {  // N rows x 8 chunks
                    const int b = c >> 3, kc = c & 7;
                    const int col = x.kt * kTcKCols + 8 * kc;
                    unsigned char* dst = bs + tc_core_off(b, kc);
                    if (b < p.batch && col < p.cols)
                        cp_async16(dst, p.xk + static_cast<size_t>(b) * p.cols + col);
                    else
                        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
            cp_async_commit();  // one group per position, empty past the end
        };

        // Register rings of 4 slots, unrolled 4 times so that every slot is a
        // fixed register (a copy between slots would wait for a load still in
        // flight): slot q % 4 holds the indices and map bytes of position q
        // (loaded at step q - 4) and the words of position q (looked up at
        // step q - 2).
        uint32_t IV[4], MV[4], W[4][2];
        Pos pd = first();  // position decoded at this step
        Pos pb = pd;       // position whose activations are copied (q + 2)
        Pos pl = pd;       // position whose indices are loaded (q + 4)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            load_ix(pl, IV[k], MV[k]);
            pl = next(pl);
        }
        words(IV[0], W[0]);
        words(IV[1], W[1]);
        issue_b(pb, 0);
        pb = next(pb);
        issue_b(pb, 1);
        pb = next(pb);
        auto step = [&](int q, uint32_t& iv_w, uint32_t (&w_w)[2], uint32_t (&w_d)[2], uint32_t& mv_d, uint32_t& iv_l,
                        uint32_t& mv_l) {
            words(iv_w, w_w);  // position q + 2
            issue_b(pb, q + 2);
            pb = next(pb);
            const int s = q % kTcStages;
            unsigned char* a = stages + s * tc_stage_bytes(N);
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // A: 2 groups of the row, position q
                const uint2 rb = s_root[(mv_d >> (8 * j)) & 0xFFu];  // R + 2 bytewise; entry 0: +2 everywhere
                const unsigned lo = (w_d[j] & 0x0F0F0F0Fu) + rb.x, hi = ((w_d[j] >> 4) & 0x0F0F0F0Fu) + rb.y;
                uint4 o;  // fp16 1024 + (P + 10) - 1034 = P, pairs in column order
                o.x = hsub2_bits(prmt(lo, hi, 0x8480u) | 0x64006400u, 0x640A640Au);
                o.y = hsub2_bits(prmt(lo, hi, 0x8581u) | 0x64006400u, 0x640A640Au);
                o.z = hsub2_bits(prmt(lo, hi, 0x8682u) | 0x64006400u, 0x640A640Au);
                o.w = hsub2_bits(prmt(lo, hi, 0x8783u) | 0x64006400u, 0x640A640Au);
                *reinterpret_cast<uint4*>(a + tc_core_off(r_l, gq + j)) = o;
            }
            load_ix(pl, iv_l, mv_l);  // position q + 4, into the slot just decoded
            pl = next(pl);
            cp_async_wait_group2();  // this position's copy (the two later ones may still run)
            fence_proxy_async_smem();  // this thread's stage writes, visible to the tensor cores
            mbar_arrive(&s_full[s]);
            pd = next(pd);
        };
        for (int q = 0; pd.u < nunits; q += 4) {
            step(q, IV[2], W[2], W[0], MV[0], IV[0], MV[0]);
            if (pd.u >= nunits) break;
            step(q + 1, IV[3], W[3], W[1], MV[1], IV[1], MV[1]);
            if (pd.u >= nunits) break;
            step(q + 2, IV[0], W[0], W[2], MV[2], IV[2], MV[2]);
            if (pd.u >= nunits) break;
            step(q + 3, IV[1], W[1], W[3], MV[3], IV[3], MV[3]);
        }
        cp_async_wait_all();
    } else if (warp == kTcMmaWarp) {
        // ------------------------------------------------------ MMA issue
        if (lane == 0) {
            constexpr uint32_t idesc = tc_idesc(N);
            int q = 0, i = 0;
            for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
                const TcUnit U = tc_unit(p, u);
                const int ab = i & 1;
                if (i >= 2) err |= tc_wait(&s_acce[ab], static_cast<unsigned>((i >> 1) - 1) & 1u);  // epilogue done
                tc_fence_after_sync();
                const uint32_t d = tmem + static_cast<uint32_t>(ab) * kAcc;
                for (int kt = U.k0; kt < U.k1; ++kt, ++q) {
                    const int s = q % kTcStages;
                    err |= tc_wait(&s_full[s], static_cast<unsigned>(q / kTcStages) & 1u);
                    tc_fence_after_sync();
                    const uint32_t a0 = smem_addr(stages + s * tc_stage_bytes(N));
                    const uint32_t b0 = a0 + static_cast<uint32_t>(kTcABytes);
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // K = 16: chunks 2k and 2k + 1, 256 bytes per step
                        umma_f16(d, tc_sdesc(a0 + 256u * k), tc_sdesc(b0 + 256u * k), idesc, kt > U.k0 || k > 0);
                    umma_commit(&s_empty[s]);
                }
                umma_commit(&s_accf[ab]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;  // tensor-memory lanes 32 quarter .. + 31
        int i = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
            const TcUnit U = tc_unit(p, u);
            const int ab = i & 1;
            err |= tc_wait(&s_accf[ab], static_cast<unsigned>(i >> 1) & 1u);
            tc_fence_after_sync();
            const int r = U.rt * kTcRows + 32 * quarter + lane;
            float* dst = p.part + (static_cast<size_t>(U.split) * p.rows + (r < p.rows ? r : 0)) * p.batch;
#pragma unroll 1
            for (int c = 0; c < N; c += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + static_cast<uint32_t>(ab) * kAcc + (static_cast<uint32_t>(32 * quarter) << 16) +
                              static_cast<uint32_t>(c),
                          v);
                if (r < p.rows) {
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        if (c + k < p.batch) dst[c + k] = __uint_as_float(v[k]);
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&s_acce[ab]);
        }
    }
    if (err) atomicOr(&g_tc_err, 1ull);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kTcMmaWarp) tmem_dealloc(tmem, kCols);
}

}  // namespace e8q
