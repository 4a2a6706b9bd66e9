// libe8q: C ABI entry points (include/e8q.h) over the sm_100a kernels.
// Argument checks, per-device constant tables, workspace sizing, launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/e8q.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode_fast.cuh"
#include "encode.cuh"
#include "encode_fast.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "ste.cuh"
#include "tables.h"

namespace e8q {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_ready[kMaxDevices];
int g_sms[kMaxDevices];

e8q_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? E8Q_OK : E8Q_ERR_CUDA; }

e8q_status ensure_device(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return E8Q_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return E8Q_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ready[dev]) {
        const HostTables* t = host_tables();
        if (!t) return E8Q_ERR_UNSUPPORTED;
        std::vector<uint2> core(65536), roots(240);
        std::memcpy(core.data(), t->core.data(), 65536 * 8);
        std::memcpy(roots.data(), t->roots.data(), 240 * 8);
        e8q_status st = E8Q_OK;
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_t1, t->t1.data(), t->t1.size() * sizeof(uint16_t)));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_t2, t->t2.data(), t->t2.size() * sizeof(uint16_t)));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_core8, core.data(), core.size() * sizeof(uint2)));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_root8, roots.data(), roots.size() * sizeof(uint2)));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_rootkey, t->root_of_key.data(), 512));
        if (st == E8Q_OK && (t->res.size() != static_cast<size_t>(kExtPoints) || t->t1e.size() != 2 * 10000 * 12 ||
                             t->t2e.size() != 2 * 10000))
            st = E8Q_ERR_UNSUPPORTED;
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_t1e, t->t1e.data(), t->t1e.size() * 4));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_t2e, t->t2e.data(), t->t2e.size() * 4));
        if (st == E8Q_OK) st = cuda_ok(cudaMemcpyToSymbol(g_res, t->res.data(), t->res.size() * 4));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_encode<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(
                cudaFuncSetAttribute(k_encode<kMaxMats>, cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(
                cudaFuncSetAttribute(k_encode_fast<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kFastSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_encode_fast<kMaxMats>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kFastSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_encode_fast<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kFastSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_encode_fast<kMaxMats, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kFastSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, kTileMaxElems * 4));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_decode_fast<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(decode_fast_smem_bytes(false))));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_decode_fast<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(decode_fast_smem_bytes(true))));
        if (st == E8Q_OK) {
            // GEMV codeword words: nibble i = P_i + 8
            std::vector<uint32_t> words(65536);
            for (int k = 0; k < 65536; ++k) {
                uint32_t wd = 0;
                for (int i = 0; i < 8; ++i) wd |= static_cast<uint32_t>((t->core[8 * k + i] + 8) & 0xF) << (4 * i);
                words[k] = wd;
            }
            st = cuda_ok(cudaMemcpyToSymbol(g_gv_tab, words.data(), words.size() * sizeof(uint32_t)));
        }
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_main<1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_main<1, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_main<1, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_main<1, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gm_main, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(kGmSmemBytes)));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gm_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxCols * 4));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gm_prep, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gm_fin, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        // prep and finalize leave the SM configured for the main kernel's shared
        // memory, so that its CTAs can start while they are still running
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_prep, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_fin<1>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_fin<2>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_fin<4>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK)
            st = cuda_ok(cudaFuncSetAttribute(k_gv_fin<8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                              cudaSharedmemCarveoutMaxShared));
        if (st == E8Q_OK) st = cuda_ok(cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev));
        if (st != E8Q_OK) return st;
        g_ready[dev] = true;
    }
    *dev_out = dev;
    return E8Q_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel on the stream is finishing; it waits for that
// kernel's results with griddepcontrol.wait.
template <typename P>
e8q_status launch_pdl(void (*kernel)(P), int grid, int threads, size_t smem, cudaStream_t s, const P& params) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_ok(cudaLaunchKernelEx(&cfg, kernel, params));
}

// log2 of the effective RHT block, or -1 if invalid
int resolve_logb(int64_t cols, int32_t block) {
    if (block == 1) return 0;
    int64_t b = block;
    if (block == 0) {
        b = cols & -cols;
        if (b > 2048) b = 2048;
    }
    if (b < 8 || b > 2048 || (b & (b - 1)) != 0 || cols % b != 0) return -1;
    int l = 0;
    while ((int64_t{1} << l) < b) ++l;
    return l;
}

bool valid_cols(int64_t cols) { return cols >= 8 && cols % 8 == 0; }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The fast kernel takes bf16 rows whose width is a multiple of 256, with an
// RHT block of at least 256, and 16-byte aligned index / output buffers.
bool fast_path_ok(const e8q_matrix& m, int logb, int dequant) {
    if (m.in_dtype != E8Q_BF16 || m.cols % 256 != 0 || logb < 8) return false;
    if (m.rows > 0 && (!aligned(m.idx, 16) || (dequant != E8Q_DEQUANT_NONE && !aligned(m.dequant, 16)))) return false;
    return true;
}

struct TileCounts {
    int64_t generic = 0;
    int64_t fast = 0;
};

TileCounts count_tiles(const e8q_matrix* mats, int n) {
    TileCounts tc;
    for (int i = 0; i < n; ++i) {
        if (mats[i].rows <= 0 || !valid_cols(mats[i].cols) || mats[i].cols > kMaxCols) continue;
        const int c = static_cast<int>(mats[i].cols);
        tc.generic += (mats[i].rows + rows_per_tile(c) - 1) / rows_per_tile(c);
        tc.fast += (mats[i].rows + fast_rows_per_tile(c) - 1) / fast_rows_per_tile(c);
    }
    return tc;
}

// workspace: [ticket, unused, status[tiles]] then the fast kernel's
// per-CTA overflow-coordinate scratch (3 tiles x 2048 groups x 16 bytes)
size_t status_bytes(const TileCounts& tc) { return align256(16 + 8 * static_cast<size_t>(tc.generic)); }
size_t scratch_bytes(const TileCounts& tc) {
    const int64_t ctas = tc.fast < kFastMaxCtas ? tc.fast : kFastMaxCtas;
    return static_cast<size_t>(ctas) * kFastSlots * kFastTileGroups * 16;
}

e8q_status check_encoded(const e8q_encoded* m, int* logb) {
    if (!m || m->rows < 0 || !valid_cols(m->cols)) return E8Q_ERR_INVALID_ARG;
    if (m->cols > kMaxCols || m->rows > (int64_t{1} << 30)) return E8Q_ERR_UNSUPPORTED;
    *logb = resolve_logb(m->cols, m->rht_block);
    if (*logb < 0) return E8Q_ERR_INVALID_ARG;
    if (m->rows > 0 && (!m->idx || !m->scale)) return E8Q_ERR_INVALID_ARG;
    if ((m->esc_row_ptr && !m->esc) || (m->ovf_row_ptr && !m->ovf)) return E8Q_ERR_INVALID_ARG;
    if (m->esc_count < 0 || m->ovf_count < 0) return E8Q_ERR_INVALID_ARG;
    if (m->group_base < 0) return E8Q_ERR_INVALID_ARG;
    return E8Q_OK;
}


// The GEMM's plan for this matrix and batch, or false for arguments it rejects.
bool gemm_plan(const e8q_encoded* m, int32_t batch, int logb, GmGeom* g) {
    if (batch < 1 || batch > kGmMaxBatch) return false;
    *g = gm_geometry(m->rows, m->cols, batch, logb);
    return g->nunits >= 0;
}

}  // namespace
}  // namespace e8q

using namespace e8q;

extern "C" {

const char* e8q_status_string(e8q_status s) {
    switch (s) {
        case E8Q_OK: return "ok";
        case E8Q_ERR_INVALID_ARG: return "invalid argument";
        case E8Q_ERR_UNSUPPORTED: return "unsupported";
        case E8Q_ERR_CUDA: return "cuda error";
        case E8Q_ERR_WORKSPACE: return "workspace too small";
        case E8Q_ERR_SCRATCH_LIMIT: return "problem too large for the built-in scratch of e8q_project_encode_noalloc";
    }
    return "unknown status";
}

e8q_status e8q_init(void) {
    int dev;
    return ensure_device(&dev);
}

e8q_status e8q_core_table(int8_t* out_coord2) {
    if (!out_coord2) return E8Q_ERR_INVALID_ARG;
    const HostTables* t = host_tables();
    if (!t) return E8Q_ERR_UNSUPPORTED;
    std::memcpy(out_coord2, t->core.data(), t->core.size());
    return E8Q_OK;
}

e8q_status e8q_escape_lookup(const int8_t* coord2, int64_t n, uint32_t* out) {
    if (n < 0 || (n > 0 && (!coord2 || !out))) return E8Q_ERR_INVALID_ARG;
    const HostTables* t = host_tables();
    if (!t) return E8Q_ERR_UNSUPPORTED;
    for (int64_t k = 0; k < n; ++k) {
        int P[8];
        for (int i = 0; i < 8; ++i) P[i] = coord2[8 * k + i];
        const uint32_t r = ext_rank(*t, P);
        out[k] = r == kExtNone ? (2u << 24) : t->res[r];
    }
    return E8Q_OK;
}

size_t e8q_encode_workspace_bytes(const e8q_matrix* mats, int32_t n_mats) {
    TileCounts tc;
    if (mats && n_mats > 0) tc = count_tiles(mats, n_mats);
    return status_bytes(tc) + scratch_bytes(tc);
}

e8q_status e8q_project_encode(const e8q_matrix* mats, int32_t n_mats, const e8q_encode_args* a, void* ws,
                              size_t ws_bytes, e8q_stream stream) {
    if (!mats || !a || n_mats < 1) return E8Q_ERR_INVALID_ARG;
    if (n_mats > kMaxMats) return E8Q_ERR_UNSUPPORTED;
    if (!a->counters || !(a->kappa > 0.f) || !std::isfinite(a->kappa)) return E8Q_ERR_INVALID_ARG;
    if (a->dequant < E8Q_DEQUANT_NONE || a->dequant > E8Q_DEQUANT_ORIGINAL) return E8Q_ERR_INVALID_ARG;
    if (a->esc_cap < 0 || a->ovf_cap < 0 || (a->esc_cap > 0 && (!a->esc || !aligned(a->esc, 8))) ||
        (a->ovf_cap > 0 && (!a->ovf || !aligned(a->ovf, 4))))
        return E8Q_ERR_INVALID_ARG;
    if (a->scale_in != 0 && a->scale_in != 1) return E8Q_ERR_INVALID_ARG;
    if ((a->flags & ~(E8Q_ENCODE_CORE_ONLY | E8Q_ENCODE_SHAPE_GAIN)) != 0 || a->reserved != 0 ||
        a->flags == (E8Q_ENCODE_CORE_ONLY | E8Q_ENCODE_SHAPE_GAIN))
        return E8Q_ERR_INVALID_ARG;

    static thread_local EncodeParams<kMaxMats> P;  // ~28 KB: keep it off the stack
    std::memset(&P, 0, sizeof(P));
    bool fast = (a->flags & E8Q_ENCODE_CORE_ONLY) == 0;  // the core-clipped projection runs in the general kernel
    for (int i = 0; i < n_mats; ++i) {
        const int logb = resolve_logb(mats[i].cols, mats[i].rht_block);
        if (!valid_cols(mats[i].cols) || mats[i].cols > kMaxCols || logb < 0 ||
            !fast_path_ok(mats[i], logb, a->dequant))
            fast = false;
    }
    int64_t tiles = 0, rows_total = 0, groups_total = 0;
    for (int i = 0; i < n_mats; ++i) {
        const e8q_matrix& m = mats[i];
        if (m.rows < 0 || !valid_cols(m.cols)) return E8Q_ERR_INVALID_ARG;
        if (m.cols > kMaxCols) return E8Q_ERR_UNSUPPORTED;
        const int logb = resolve_logb(m.cols, m.rht_block);
        if (logb < 0) return E8Q_ERR_INVALID_ARG;
        if (m.in_dtype != E8Q_F32 && m.in_dtype != E8Q_BF16) return E8Q_ERR_INVALID_ARG;
        if (m.rows > 0) {
            if (!m.w || !m.signs || !m.idx || !m.scale) return E8Q_ERR_INVALID_ARG;
            if (!aligned(m.w, 16) || !aligned(m.signs, 8) || !aligned(m.idx, 2) || !aligned(m.scale, 4))
                return E8Q_ERR_INVALID_ARG;
            if (a->dequant != E8Q_DEQUANT_NONE && (!m.dequant || !aligned(m.dequant, 16))) return E8Q_ERR_INVALID_ARG;
        }
        const int rpt = fast ? fast_rows_per_tile(static_cast<int>(m.cols)) : rows_per_tile(static_cast<int>(m.cols));
        MatDesc& d = P.m[i];
        d.w = m.w;
        d.signs = m.signs;
        d.idx = m.idx;
        d.scale = m.scale;
        d.dq = m.dequant;
        d.rows = static_cast<int32_t>(m.rows);
        d.cols = static_cast<int32_t>(m.cols);
        d.meta = logb | ((m.in_dtype == E8Q_BF16) ? 16 : 0) | (rpt << 8);
        d.tile_base = static_cast<int32_t>(tiles);
        d.row_base = static_cast<int32_t>(rows_total);
        d.group_base = static_cast<uint32_t>(groups_total);
        tiles += (m.rows + rpt - 1) / rpt;
        rows_total += m.rows;
        groups_total += m.rows * (m.cols / 8);
        if (groups_total >= (int64_t{1} << 31) || rows_total >= (int64_t{1} << 31)) return E8Q_ERR_UNSUPPORTED;
    }
    const TileCounts tc = count_tiles(mats, n_mats);
    const size_t need = status_bytes(tc) + scratch_bytes(tc);
    if (!ws || ws_bytes < need || !aligned(ws, 256)) return E8Q_ERR_WORKSPACE;

    int dev;
    e8q_status st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = cuda_ok(cudaMemsetAsync(a->counters, 0, sizeof(e8q_counters), s));
    if (st == E8Q_OK) st = cuda_ok(cudaMemsetAsync(ws, 0, 16 + 8 * static_cast<size_t>(tiles), s));
    if (st != E8Q_OK) return st;
    if (tiles == 0) {  // nothing to encode: empty CSR
        if (a->esc_row_ptr) st = cuda_ok(cudaMemsetAsync(a->esc_row_ptr + rows_total, 0, sizeof(int64_t), s));
        if (st == E8Q_OK && a->ovf_row_ptr)
            st = cuda_ok(cudaMemsetAsync(a->ovf_row_ptr + rows_total, 0, sizeof(int64_t), s));
        return st;
    }
    P.esc = a->esc;
    P.ovf = a->ovf;
    P.esc_rp = a->esc_row_ptr;
    P.ovf_rp = a->ovf_row_ptr;
    P.ctr = a->counters;
    P.ws = static_cast<unsigned long long*>(ws);
    P.esc_cap = a->esc_cap;
    P.ovf_cap = a->ovf_cap;
    P.kappa = a->kappa;
    P.dq_mode = a->dequant;
    P.scale_in = a->scale_in;
    P.n_mats = n_mats;
    P.n_tiles = static_cast<int32_t>(tiles);
    P.total_rows = static_cast<int32_t>(rows_total);
    P.core_only = (a->flags & E8Q_ENCODE_CORE_ONLY) ? 1 : 0;
    P.shape_gain = (a->flags & E8Q_ENCODE_SHAPE_GAIN) ? 1 : 0;
    {  // |2x| <= 2 kappa sqrt(cols): clamp coordinates only when that could pass 2^14
        int64_t maxc = 0;
        for (int i = 0; i < n_mats; ++i) maxc = mats[i].cols > maxc ? mats[i].cols : maxc;
        P.clamp = (a->scale_in != 0 || 2.0 * a->kappa * std::sqrt(static_cast<double>(maxc)) > 16384.0) ? 1 : 0;
    }
    if (fast) {
        int64_t g = tiles < g_sms[dev] ? tiles : g_sms[dev];
        if (g > kFastMaxCtas) g = kFastMaxCtas;
        const int grid = static_cast<int>(g);
        int16_t* scratch = reinterpret_cast<int16_t*>(static_cast<char*>(ws) + status_bytes(tc));
        if (n_mats == 1) {
            EncodeParams<1> P1;
            std::memcpy(&P1, &P, offsetof(EncodeParams<1>, m));
            P1.m[0] = P.m[0];
            if (P.shape_gain)
                k_encode_fast<1, true><<<grid, kFastThreads, kFastSmemBytes, s>>>(P1, scratch);
            else
                k_encode_fast<1><<<grid, kFastThreads, kFastSmemBytes, s>>>(P1, scratch);
        } else if (P.shape_gain) {
            k_encode_fast<kMaxMats, true><<<grid, kFastThreads, kFastSmemBytes, s>>>(P, scratch);
        } else {
            k_encode_fast<kMaxMats><<<grid, kFastThreads, kFastSmemBytes, s>>>(P, scratch);
        }
        return cuda_ok(cudaGetLastError());
    }
    const int grid = static_cast<int>(tiles < g_sms[dev] ? tiles : g_sms[dev]);
    if (n_mats == 1) {
        EncodeParams<1> P1;
        std::memcpy(&P1, &P, offsetof(EncodeParams<1>, m));
        P1.m[0] = P.m[0];
        k_encode<1><<<grid, kEncThreads, kEncSmemBytes, s>>>(P1);
    } else {
        k_encode<kMaxMats><<<grid, kEncThreads, kEncSmemBytes, s>>>(P);
    }
    return cuda_ok(cudaGetLastError());
}

e8q_status e8q_decode(const e8q_encoded* m, int32_t basis, void* out_bf16, e8q_stream stream) {
    int logb;
    e8q_status st = check_encoded(m, &logb);
    if (st != E8Q_OK) return st;
    if (basis != E8Q_DEQUANT_ROTATED && basis != E8Q_DEQUANT_ORIGINAL) return E8Q_ERR_INVALID_ARG;
    if (m->rows == 0) return E8Q_OK;
    if (!out_bf16 || !aligned(out_bf16, 16)) return E8Q_ERR_INVALID_ARG;
    if (basis == E8Q_DEQUANT_ORIGINAL && (!m->signs || !aligned(m->signs, 8))) return E8Q_ERR_INVALID_ARG;
    if (m->esc_row_ptr && !aligned(m->esc, 8)) return E8Q_ERR_INVALID_ARG;
    int dev;
    st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    DecodeParams p;
    p.idx = m->idx;
    p.scale = m->scale;
    p.signs = m->signs;
    p.esc = m->esc;
    p.esc_rp = m->esc_row_ptr;
    p.ovf = m->ovf;
    p.ovf_rp = m->ovf_row_ptr;
    p.esc_n = m->esc_row_ptr ? m->esc_count : 0;
    p.ovf_n = m->ovf_row_ptr ? m->ovf_count : 0;
    p.out = static_cast<uint16_t*>(out_bf16);
    p.group_base = m->group_base;
    p.rows = static_cast<int32_t>(m->rows);
    p.cols = static_cast<int32_t>(m->cols);
    p.logb = logb;
    p.basis = basis;
    // fast path (original basis through the register Hadamard, B >= 256); its
    // staging warp copies indices in 16-byte words and overflow group ids in
    // 4-byte words
    const bool orig = basis == E8Q_DEQUANT_ORIGINAL;
    if (p.cols % 256 == 0 && (!orig || logb >= 8) && (reinterpret_cast<uintptr_t>(p.idx) & 15) == 0 &&
        (reinterpret_cast<uintptr_t>(p.ovf) & 3) == 0) {
        p.rpt = decode_fast_rows_per_tile(p.cols);
        p.n_tiles = (p.rows + p.rpt - 1) / p.rpt;
        const int per_sm = orig ? kDfCtasOrig : kDfCtasRot;
        const int grid = p.n_tiles < per_sm * g_sms[dev] ? p.n_tiles : per_sm * g_sms[dev];
        if (orig)
            k_decode_fast<true><<<grid, kDfThreads, decode_fast_smem_bytes(true), reinterpret_cast<cudaStream_t>(stream)>>>(p);
        else
            k_decode_fast<false>
                <<<grid, kDfThreads, decode_fast_smem_bytes(false), reinterpret_cast<cudaStream_t>(stream)>>>(p);
        return cuda_ok(cudaGetLastError());
    }
    p.rpt = rows_per_tile(p.cols);
    p.n_tiles = (p.rows + p.rpt - 1) / p.rpt;
    const int grid = p.n_tiles < 2 * g_sms[dev] ? p.n_tiles : 2 * g_sms[dev];
    k_decode<<<grid, kDecThreads, kTileMaxElems * 4, reinterpret_cast<cudaStream_t>(stream)>>>(p);
    return cuda_ok(cudaGetLastError());
}

size_t e8q_gemv_workspace_bytes(const e8q_encoded* m, int32_t batch) {
    if (!m || m->rows < 0 || m->cols <= 0 || m->cols > kMaxCols || batch <= 0 || batch > 256) return 256;
    const GvGeom g = gv_geometry(m->rows, m->cols, batch, 0, kGvMaxCtas);
    return gv_workspace(g).total;
}

e8q_status e8q_dequant_gemv(const e8q_encoded* m, const void* x_bf16, int32_t batch, void* y_bf16, void* ws,
                            size_t ws_bytes, e8q_stream stream) {
    int logb;
    e8q_status st = check_encoded(m, &logb);
    if (st != E8Q_OK) return st;
    if (batch < 1 || batch > 256) return E8Q_ERR_INVALID_ARG;
    if (!x_bf16 || !y_bf16 || !m->signs || !aligned(x_bf16, 16) || !aligned(y_bf16, 2)) return E8Q_ERR_INVALID_ARG;
    if (m->esc_row_ptr && !aligned(m->esc, 8)) return E8Q_ERR_INVALID_ARG;
    const size_t need = e8q_gemv_workspace_bytes(m, batch);
    if (!ws || ws_bytes < need || !aligned(ws, 256)) return E8Q_ERR_WORKSPACE;
    if (m->rows == 0) return E8Q_OK;
    int dev;
    st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int ctas = g_sms[dev] < kGvMaxCtas ? g_sms[dev] : kGvMaxCtas;
    const GvGeom g = gv_geometry(m->rows, m->cols, batch, logb, ctas);
    const GvWs L = gv_workspace(g);
    unsigned char* w = static_cast<unsigned char*>(ws);
    const bool has_esc = m->esc_row_ptr != nullptr;

    GvPrepParams pp;
    pp.x = static_cast<const uint16_t*>(x_bf16);
    pp.signs = m->signs;
    pp.x32 = reinterpret_cast<float*>(w + L.x32);
    pp.x16 = reinterpret_cast<uint4*>(w + L.x16);
    pp.xe = reinterpret_cast<float*>(w + L.xe);
    pp.esc = m->esc;
    pp.esc_rp = m->esc_row_ptr;
    pp.map = reinterpret_cast<uint8_t*>(w + L.map);
    pp.esc_n = has_esc ? m->esc_count : 0;
    pp.group_base = m->group_base;
    pp.g = g;
    pp.n_xcta = g.nseg * batch;
    const int n_ecta = has_esc ? (g.rows + 7) / 8 : 0;
    k_gv_prep<<<pp.n_xcta + n_ecta, 256, 0, s>>>(pp);
    st = cuda_ok(cudaGetLastError());
    if (st != E8Q_OK) return st;

    GvMainParams mp;
    mp.idx = m->idx;
    mp.x16 = pp.x16;
    mp.map = has_esc ? pp.map : nullptr;
    mp.part = reinterpret_cast<float*>(w + L.part);
    mp.g = g;
    mp.vec_idx = (g.gpr % 8 == 0 && aligned(m->idx, 16)) ? 1 : 0;
    const int grid = g.nctas;
    for (int v0 = 0; v0 < g.nbt; v0 += kGvPassTiles) {
        const int nt = g.nbt - v0 < kGvPassTiles ? g.nbt - v0 : kGvPassTiles;
        mp.v0 = v0;
        // one 16-row tile per warp, 16 warps (two tiles on 8 warps measured slower at batch 64 and 256)
        if (nt == 1) st = launch_pdl(k_gv_main<1, 1>, grid, 512, kGvSmemBytes, s, mp);
        else if (nt == 2) st = launch_pdl(k_gv_main<1, 2>, grid, 512, kGvSmemBytes, s, mp);
        else if (nt <= 4) st = launch_pdl(k_gv_main<1, 4>, grid, 512, kGvSmemBytes, s, mp);
        else st = launch_pdl(k_gv_main<1, 8>, grid, 512, kGvSmemBytes, s, mp);
        if (st != E8Q_OK) return st;
    }

    GvFinParams fp;
    fp.part = mp.part;
    fp.xe = pp.xe;
    fp.x32 = pp.x32;
    fp.scale = m->scale;
    fp.ovf = m->ovf;
    fp.ovf_rp = m->ovf_row_ptr;
    fp.y = static_cast<uint16_t*>(y_bf16);
    fp.ovf_n = m->ovf_row_ptr ? m->ovf_count : 0;
    fp.group_base = m->group_base;
    fp.g = g;
    fp.bl_log = 0;
    while ((1 << fp.bl_log) < batch && fp.bl_log < 5) ++fp.bl_log;
    const int kb = (batch + 31) / 32;  // batch rows per lane
    const int fgrid = (g.rows + 7) / 8;
    if (kb == 1) return launch_pdl(k_gv_fin<1>, fgrid, 256, 0, s, fp);
    if (kb == 2) return launch_pdl(k_gv_fin<2>, fgrid, 256, 0, s, fp);
    if (kb <= 4) return launch_pdl(k_gv_fin<4>, fgrid, 256, 0, s, fp);
    return launch_pdl(k_gv_fin<8>, fgrid, 256, 0, s, fp);
}

size_t e8q_gemm_workspace_bytes(const e8q_encoded* m, int32_t batch) {
    int logb;
    GmGeom g;
    if (check_encoded(m, &logb) != E8Q_OK || !gemm_plan(m, batch, logb, &g)) return 256;
    return gm_workspace(g).total;
}

e8q_status e8q_dequant_gemm(const e8q_encoded* m, const void* x_bf16, int32_t batch, void* y_bf16, void* ws,
                            size_t ws_bytes, e8q_stream stream) {
    int logb;
    e8q_status st = check_encoded(m, &logb);
    if (st != E8Q_OK) return st;
    if (batch < 1 || batch > kGmMaxBatch) return E8Q_ERR_INVALID_ARG;
    if (!x_bf16 || !y_bf16 || !m->signs || !aligned(x_bf16, 16) || !aligned(y_bf16, 2)) return E8Q_ERR_INVALID_ARG;
    if (m->esc_row_ptr && !aligned(m->esc, 8)) return E8Q_ERR_INVALID_ARG;
    if (m->ovf_row_ptr && !aligned(m->ovf, 4)) return E8Q_ERR_INVALID_ARG;
    GmGeom g;
    if (!gemm_plan(m, batch, logb, &g)) return E8Q_ERR_UNSUPPORTED;
    const GmWs L = gm_workspace(g);
    if (!ws || ws_bytes < L.total || !aligned(ws, 256)) return E8Q_ERR_WORKSPACE;
    if (m->rows == 0) return E8Q_OK;
    int dev;
    st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* w = static_cast<unsigned char*>(ws);

    GmPrepParams pp;
    pp.x = static_cast<const uint16_t*>(x_bf16);
    pp.signs = m->signs;
    pp.img = w + L.img;
    pp.xe = reinterpret_cast<float*>(w + L.xe);
    pp.esc = m->esc;
    pp.esc_rp = m->esc_row_ptr;
    pp.esc_n = m->esc_row_ptr ? m->esc_count : 0;
    pp.ovf = m->ovf;
    pp.ovf_rp = m->ovf_row_ptr;
    pp.ovf_n = m->ovf_row_ptr ? m->ovf_count : 0;
    pp.map = reinterpret_cast<uint16_t*>(w + L.map);
    pp.farf = w + L.farf;
    pp.err = reinterpret_cast<unsigned long long*>(w + L.err);
    pp.group_base = m->group_base;
    pp.g = g;
    pp.n_xcta = (batch + 15) / 16 * 16;
    const int n_rcta = (g.rows + 7) / 8;
    k_gm_prep<<<pp.n_xcta + n_rcta, 256, static_cast<size_t>(g.cols) * 4, s>>>(pp);
    st = cuda_ok(cudaGetLastError());
    if (st != E8Q_OK) return st;

    GmMainParams mp;
    mp.idx = m->idx;
    mp.map = pp.map;
    mp.img = pp.img;
    mp.xe = pp.xe;
    mp.scale = m->scale;
    mp.farf = pp.farf;
    mp.ovf = m->ovf;
    mp.ovf_rp = m->ovf_row_ptr;
    mp.ovf_n = pp.ovf_n;
    mp.part = reinterpret_cast<float*>(w + L.part);
    mp.y = static_cast<uint16_t*>(y_bf16);
    mp.err = pp.err;
    mp.group_base = m->group_base;
    mp.g = g;
    const int grid = g.nunits < g_sms[dev] ? g.nunits : g_sms[dev];
    st = launch_pdl(k_gm_main, grid, kGmThreads, kGmSmemBytes, s, mp);
    if (st != E8Q_OK || g.nsplit == 1) return st;

    GmFinParams fp;
    fp.part = mp.part;
    fp.xe = pp.xe;
    fp.scale = m->scale;
    fp.farf = pp.farf;
    fp.img = pp.img;
    fp.ovf = m->ovf;
    fp.ovf_rp = m->ovf_row_ptr;
    fp.ovf_n = pp.ovf_n;
    fp.group_base = m->group_base;
    fp.y = mp.y;
    fp.g = g;
    const size_t n = static_cast<size_t>(batch) * g.rows;
    const size_t fb = (n + 255) / 256;
    const int fgrid = static_cast<int>(fb < static_cast<size_t>(16 * g_sms[dev]) ? fb : 16 * g_sms[dev]);
    return launch_pdl(k_gm_fin, fgrid, 256, 0, s, fp);
}

e8q_status e8q_ste_backward(const void* grad_dequant, void* grad_latent, int64_t n, e8q_stream stream) {
    if (n < 0) return E8Q_ERR_INVALID_ARG;
    if (n == 0) return E8Q_OK;
    if (!grad_dequant || !grad_latent || !aligned(grad_dequant, 2) || !aligned(grad_latent, 2))
        return E8Q_ERR_INVALID_ARG;
    if (grad_dequant == grad_latent) return E8Q_OK;  // the identity, aliased: nothing to move
    const uintptr_t a = reinterpret_cast<uintptr_t>(grad_dequant), b = reinterpret_cast<uintptr_t>(grad_latent);
    const uintptr_t bytes = static_cast<uintptr_t>(n) * 2;
    if (a < b + bytes && b < a + bytes) return E8Q_ERR_INVALID_ARG;  // partial overlap
    int dev;
    e8q_status st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int grid = 4 * g_sms[dev];  // persistent grid: 4 CTAs of 512 threads an SM
    if (aligned(grad_dequant, 16) && aligned(grad_latent, 16)) {
        const long long n16 = n / 8;
        if (n16 > 0)
            k_ste_copy16<<<grid, kSteThreads, 0, s>>>(static_cast<const uint4*>(grad_dequant),
                                                      static_cast<uint4*>(grad_latent), n16);
        const long long tail = n - 8 * n16;
        if (tail > 0)
            k_ste_copy2<<<1, kSteThreads, 0, s>>>(static_cast<const uint16_t*>(grad_dequant) + 8 * n16,
                                                  static_cast<uint16_t*>(grad_latent) + 8 * n16, tail);
    } else {
        k_ste_copy2<<<grid, kSteThreads, 0, s>>>(static_cast<const uint16_t*>(grad_dequant),
                                                 static_cast<uint16_t*>(grad_latent), n);
    }
    return cuda_ok(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------------
// Encode with a built-in scratch (no allocation by the library or caller)
// ---------------------------------------------------------------------
namespace e8q {
namespace {
// Ticket and tile-status words of the encode kernel, for callers that cannot
// allocate.  Host code must not pass this name to a kernel: on the host it is
// only a stand-in; the device address comes from cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = size_t{2} << 20;
static __device__ __align__(256) unsigned long long g_noalloc_scratch[kNoAllocScratchBytes / 8];
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];
}  // namespace
}  // namespace e8q

extern "C" e8q_status e8q_project_encode_noalloc(const e8q_matrix* mats, int32_t n_mats, const e8q_encode_args* a,
                                                 e8q_stream stream) {
    if (!mats || !a || n_mats < 1) return E8Q_ERR_INVALID_ARG;
    if (n_mats > kMaxMats) return E8Q_ERR_UNSUPPORTED;
    if (!a->counters || !(a->kappa > 0.f) || !std::isfinite(a->kappa)) return E8Q_ERR_INVALID_ARG;
    if (a->dequant < E8Q_DEQUANT_NONE || a->dequant > E8Q_DEQUANT_ORIGINAL) return E8Q_ERR_INVALID_ARG;
    if (a->esc_cap < 0 || a->ovf_cap < 0 || (a->esc_cap > 0 && (!a->esc || !aligned(a->esc, 8))) ||
        (a->ovf_cap > 0 && (!a->ovf || !aligned(a->ovf, 4))))
        return E8Q_ERR_INVALID_ARG;
    if (a->scale_in != 0 && a->scale_in != 1) return E8Q_ERR_INVALID_ARG;
    if ((a->flags & ~(E8Q_ENCODE_CORE_ONLY | E8Q_ENCODE_SHAPE_GAIN)) != 0 || a->reserved != 0 ||
        a->flags == (E8Q_ENCODE_CORE_ONLY | E8Q_ENCODE_SHAPE_GAIN))
        return E8Q_ERR_INVALID_ARG;

    static thread_local EncodeParams<kMaxMats> P;
    std::memset(&P, 0, sizeof(P));
    int64_t tiles = 0, rows_total = 0, groups_total = 0;
    for (int i = 0; i < n_mats; ++i) {
        const e8q_matrix& m = mats[i];
        if (m.rows < 0 || !valid_cols(m.cols)) return E8Q_ERR_INVALID_ARG;
        if (m.cols > kMaxCols) return E8Q_ERR_UNSUPPORTED;
        const int logb = resolve_logb(m.cols, m.rht_block);
        if (logb < 0) return E8Q_ERR_INVALID_ARG;
        if (m.in_dtype != E8Q_F32 && m.in_dtype != E8Q_BF16) return E8Q_ERR_INVALID_ARG;
        if (m.rows > 0) {
            if (!m.w || !m.signs || !m.idx || !m.scale) return E8Q_ERR_INVALID_ARG;
            if (!aligned(m.w, 16) || !aligned(m.signs, 8) || !aligned(m.idx, 2) || !aligned(m.scale, 4))
                return E8Q_ERR_INVALID_ARG;
            if (a->dequant != E8Q_DEQUANT_NONE && (!m.dequant || !aligned(m.dequant, 16))) return E8Q_ERR_INVALID_ARG;
        }
        const int rpt = rows_per_tile(static_cast<int>(m.cols));
        MatDesc& d = P.m[i];
        d.w = m.w;
        d.signs = m.signs;
        d.idx = m.idx;
        d.scale = m.scale;
        d.dq = m.dequant;
        d.rows = static_cast<int32_t>(m.rows);
        d.cols = static_cast<int32_t>(m.cols);
        d.meta = logb | ((m.in_dtype == E8Q_BF16) ? 16 : 0) | (rpt << 8);
        d.tile_base = static_cast<int32_t>(tiles);
        d.row_base = static_cast<int32_t>(rows_total);
        d.group_base = static_cast<uint32_t>(groups_total);
        tiles += (m.rows + rpt - 1) / rpt;
        rows_total += m.rows;
        groups_total += m.rows * (m.cols / 8);
        if (groups_total >= (int64_t{1} << 31) || rows_total >= (int64_t{1} << 31)) return E8Q_ERR_UNSUPPORTED;
    }
    const size_t need = 16 + 8 * static_cast<size_t>(tiles);
    if (need > kNoAllocScratchBytes) return E8Q_ERR_SCRATCH_LIMIT;

    int dev;
    e8q_status st = ensure_device(&dev);
    if (st != E8Q_OK) return st;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_addr[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return E8Q_ERR_CUDA;
            g_noalloc_addr[dev] = p;
        }
        scratch = g_noalloc_addr[dev];
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = cuda_ok(cudaMemsetAsync(a->counters, 0, sizeof(e8q_counters), s));
    if (st == E8Q_OK) st = cuda_ok(cudaMemsetAsync(scratch, 0, need, s));
    if (st != E8Q_OK) return st;
    if (tiles == 0) {
        if (a->esc_row_ptr) st = cuda_ok(cudaMemsetAsync(a->esc_row_ptr + rows_total, 0, sizeof(int64_t), s));
        if (st == E8Q_OK && a->ovf_row_ptr)
            st = cuda_ok(cudaMemsetAsync(a->ovf_row_ptr + rows_total, 0, sizeof(int64_t), s));
        return st;
    }
    P.esc = a->esc;
    P.ovf = a->ovf;
    P.esc_rp = a->esc_row_ptr;
    P.ovf_rp = a->ovf_row_ptr;
    P.ctr = a->counters;
    P.ws = static_cast<unsigned long long*>(scratch);
    P.esc_cap = a->esc_cap;
    P.ovf_cap = a->ovf_cap;
    P.kappa = a->kappa;
    P.dq_mode = a->dequant;
    P.scale_in = a->scale_in;
    P.n_mats = n_mats;
    P.n_tiles = static_cast<int32_t>(tiles);
    P.total_rows = static_cast<int32_t>(rows_total);
    P.core_only = (a->flags & E8Q_ENCODE_CORE_ONLY) ? 1 : 0;
    P.shape_gain = (a->flags & E8Q_ENCODE_SHAPE_GAIN) ? 1 : 0;
    const int grid = static_cast<int>(tiles < g_sms[dev] ? tiles : g_sms[dev]);
    if (n_mats == 1) {
        EncodeParams<1> P1;
        std::memcpy(&P1, &P, offsetof(EncodeParams<1>, m));
        P1.m[0] = P.m[0];
        k_encode<1><<<grid, kEncThreads, kEncSmemBytes, s>>>(P1);
    } else {
        k_encode<kMaxMats><<<grid, kEncThreads, kEncSmemBytes, s>>>(P);
    }
    return cuda_ok(cudaGetLastError());
}

