/*
 * e8q.h -- C ABI of libe8q, the B200 (sm_100a) library for the 2-bit
 * E8-lattice quantize path.
 *
 * What the path computes follows "E8-QAT: Efficient 2-Bit
 * Quantization-Aware Training with Implicit Lattice Codebooks":
 *   - abstract: E8 is an implicit 8-dimensional codebook; weight groups are
 *     projected onto it by arithmetic, with no stored codebook searched; a
 *     2-bit core encoding plus a sparse extension keeps every selected
 *     lattice point exactly; decoding from the 2-bit form is the inference
 *     path whose throughput the paper compares with BF16;
 *   - Figure 2 caption: latent weights start in a fixed E8 core; projection
 *     with an identity straight-through estimator (STE) during training;
 *     core indices plus sparse escape records; Hadamard transforms and
 *     reconstruction scales around the projection;
 *   - appendix Table 3: the core has 65,536 codewords; every escaped
 *     group's residual is one element of the root set R (240 roots);
 *   - appendix Table 10: payload b = 2 + 20*rho bits per weight with
 *     20-byte coordinate records (rho = escaped fraction of groups).
 *
 * Conventions fixed here where the pages are silent:
 *   - Weights: row-major [rows][cols]; a group is 8 consecutive columns of
 *     one row; cols % 8 == 0.
 *   - RHT: u = d (.) w with d in {+1,-1}^cols (one vector per matrix), then
 *     v = H_B u / sqrt(B) on every B-wide block of a row, H_B the Sylvester
 *     Hadamard matrix in natural order (H[i][j] = (-1)^popcount(i & j)).
 *     Default B = largest power of two dividing cols, capped at 2048.
 *   - Scale: s_r = sqrt(mean_c v_rc^2) / kappa, stored as fp32; x = v / s_r
 *     (x = 0 when s_r = 0).  Non-finite inputs are read as 0 and counted.
 *   - Projection: nearest E8 point of each 8-group of x (Conway-Sloane D8
 *     and D8+1/2 rounding, keep the closer).  Lattice points are handled in
 *     doubled coordinates P = 2p (integers, all even or all odd, sum % 4 == 0).
 *   - Core: the 65,536 E8 points first in (|p|^2, then P lexicographically,
 *     most negative first) order; the core index of a point is its rank in
 *     that order (index 0 is the origin, 1..240 the roots).
 *   - Escape: a point outside the core that equals core point + root r is
 *     stored as idx = core index of (p - r) plus an 8-byte escape record;
 *     among several such roots the one giving the smallest core index is
 *     used.  A point with no such root gets idx = 0 and a 20-byte overflow
 *     record holding its doubled coordinates.
 *
 * Memory: every pointer argument is DEVICE memory unless marked "host".  The
 * caller owns all buffers; the library allocates nothing per call.  On the
 * first call on a device the library uploads its constant tables (about
 * 600 KB of __device__ arrays, built on the host); that first call on each
 * device must not be inside a CUDA graph capture.  e8q_init() does it
 * explicitly.
 *
 * Streams: every compute call enqueues its work on `stream` and returns
 * without waiting.  The return code covers argument checks and launch
 * errors only; conditions found in the data (escape counts, capacity
 * shortfall, non-finite inputs, a wait that gave up) are written to the
 * device-side e8q_counters (for e8q_dequant_gemm: the first word of its
 * workspace), which the caller reads after synchronising.
 */
#ifndef E8Q_H
#define E8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* e8q_stream;

typedef enum {
    E8Q_OK = 0,
    E8Q_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or enum */
    E8Q_ERR_UNSUPPORTED = 2, /* valid but outside the library's limits */
    E8Q_ERR_CUDA = 3,        /* a CUDA call or launch failed */
    E8Q_ERR_WORKSPACE = 4,   /* workspace missing or too small */
    E8Q_ERR_SCRATCH_LIMIT = 5 /* larger than e8q_project_encode_noalloc's built-in scratch */
} e8q_status;

typedef enum { E8Q_F32 = 0, E8Q_BF16 = 1 } e8q_dtype;

typedef enum {
    E8Q_DEQUANT_NONE = 0,
    E8Q_DEQUANT_ROTATED = 1, /* bf16(s * p): the Hadamard-domain weight, rounded once */
    E8Q_DEQUANT_ORIGINAL = 2 /* bf16(d (.) H_B (s * p) / sqrt(B)): original basis (STE forward) */
} e8q_dequant_mode;

/* Escape record: core point + one root (Table 3, "single-root membership").
 * 8 bytes, little-endian. */
typedef struct e8q_escape {
    uint32_t group;   /* group id, numbered over the whole encode call */
    uint16_t core;    /* core index of p - r (also stored in idx[group]) */
    uint8_t root;     /* index of r among the 240 roots, lexicographic order */
    uint8_t reserved; /* 0 */
} e8q_escape;

/* Overflow record: a point that is not core + one root.  20 bytes, the
 * record size the E8-QAT Table 10 payload assumes. */
typedef struct e8q_overflow {
    uint32_t group;     /* group id, numbered over the whole encode call */
    int16_t coord2[8];  /* doubled coordinates 2p, clamped to int16 */
} e8q_overflow;

/* Device-side results of one encode call (written, not accumulated). */
typedef struct e8q_counters {
    unsigned long long n_escape;    /* escape records produced (may exceed esc_cap) */
    unsigned long long n_overflow;  /* overflow records produced (may exceed ovf_cap) */
    unsigned long long n_nonfinite; /* input elements that were NaN or Inf, read as 0 */
    unsigned long long n_dropped;   /* records not stored: past esc_cap / ovf_cap */
    unsigned long long n_clamped;   /* overflow coordinates outside int16 */
    unsigned long long err;         /* bit 0: an ordering wait gave up (output invalid) */
} e8q_counters;

/* One weight matrix of an encode call. */
typedef struct e8q_matrix {
    const void* w;        /* [rows][cols], in_dtype, 16-byte aligned */
    const int8_t* signs;  /* [cols], each +1 or -1 (the RHT sign vector d) */
    uint16_t* idx;        /* out: [rows][cols/8] core indices */
    float* scale;         /* out: [rows] reconstruction scales s_r */
    void* dequant;        /* out: bf16 [rows][cols], 16-byte aligned, or NULL */
    int64_t rows;         /* >= 0 */
    int64_t cols;         /* multiple of 8, 8..16384 */
    int32_t rht_block;    /* 0 = default rule, 1 = no transform, else power of two 8..2048 dividing cols */
    int32_t in_dtype;     /* e8q_dtype */
} e8q_matrix;

/* Shared arguments and outputs of an encode call. */
typedef struct e8q_encode_args {
    float kappa;               /* > 0; s_r = rms_r / kappa (1 = row RMS) */
    int32_t dequant;           /* e8q_dequant_mode for the matrices' dequant buffers */
    int32_t scale_in;          /* 0: compute s_r and write mats[].scale; 1: read s_r from
                                  mats[].scale (fixed reconstruction scales; a value that is
                                  not finite and > 0 reads as 0, giving x = 0) */
    e8q_escape* esc;           /* out: escape records sorted by group, capacity esc_cap; 8-byte aligned */
    int64_t esc_cap;
    e8q_overflow* ovf;         /* out: overflow records sorted by group, capacity ovf_cap; 4-byte aligned */
    int64_t ovf_cap;
    int64_t* esc_row_ptr;      /* out: [total_rows + 1] CSR offsets into esc, or NULL */
    int64_t* ovf_row_ptr;      /* out: [total_rows + 1] CSR offsets into ovf, or NULL */
    e8q_counters* counters;    /* out: required */
    int32_t flags;             /* E8Q_ENCODE_* bits; 0 = the projection of QAT */
    int32_t reserved;          /* 0 */
} e8q_encode_args;

/* e8q_encode_args.flags */
enum {
    /* Core-clipped projection (E8-QAT Figure 2 (a): post-training quantisation
     * initialises the latent weights from the fixed E8 core): every group
     * takes the core point nearest to x (equal distances: the smaller core
     * index) instead of the nearest E8 point, so the call writes indices only
     * and no escape or overflow record (rho = 0).  The dequant outputs are
     * those of the chosen core points. */
    E8Q_ENCODE_CORE_ONLY = 1,
    /* Shape-gain code (SQuAT page, "shape and scale split": each weight
     * vector splits into a unit direction, quantised against a spherical E8
     * codebook, and a scalar gain through a low-bit scalar quantiser).  After
     * the same sign flip, RHT and row scale, each group x gets the 16-bit
     * code k << 12 | d: d (0 .. 2159) the index, in lexicographic order, of
     * the |p|^2 = 4 shell point c of largest <x, c> (the nearest direction;
     * core index 241 + d), k = min(15, floor(|x| / (6 / 16))) the gain level.
     * The reconstruction is x-hat = (k + 1/2) (6 / 16) c / |c|; the dequant
     * outputs are those of x-hat (rotated: bf16(s x-hat); original:
     * bf16(d (.) H_B (s x-hat) / sqrt(B))).  No escape or overflow record is
     * written.  Not combinable with E8Q_ENCODE_CORE_ONLY; decode and GEMV
     * read the lattice encoding only. */
    E8Q_ENCODE_SHAPE_GAIN = 2
};

/* One encoded matrix, as read by decode and GEMV. */
typedef struct e8q_encoded {
    const uint16_t* idx;          /* [rows][cols/8] */
    const float* scale;           /* [rows] */
    const int8_t* signs;          /* [cols] (read for the original basis and the GEMV) */
    const e8q_escape* esc;        /* records of the encode call, or NULL when there are none */
    const int64_t* esc_row_ptr;   /* [rows + 1]: this matrix's rows' slice of the call's CSR */
    const e8q_overflow* ovf;
    const int64_t* ovf_row_ptr;   /* [rows + 1] */
    int64_t esc_count;            /* records readable at esc (offsets at or past it are skipped) */
    int64_t ovf_count;            /* records readable at ovf */
    int64_t rows;
    int64_t cols;
    int64_t group_base;           /* first group id of this matrix in its encode call */
    int32_t rht_block;            /* as given at encode time (0 = default rule) */
    int32_t reserved;             /* 0 */
} e8q_encoded;

/* Human-readable name of a status code.  Host only. */
const char* e8q_status_string(e8q_status s);

/* Uploads the constant tables to the current device if not done yet.
 * Synchronous; call outside graph capture.  Other calls do it on demand. */
e8q_status e8q_init(void);

/* Host only: the library's own core table, doubled coordinates [65536][8]
 * (host buffer), rank order.  Lets a CPU test compare it with other
 * decoders (Table 3, "core decoding agreement"). */
e8q_status e8q_core_table(int8_t* out_coord2);

/* Host only: how the encode kernels encode given doubled E8 points
 * (coord2: host [n][8], each a point of E8; out: host [n]).  A core point
 * gives its core index; a point outside the core gives, by the escape rule
 * (the root r maximising <p, r>, ties to the lexicographically largest r;
 * E8-QAT appendix Table 3, single-root membership), rank(p - r) |
 * (index of r << 16) | (1 << 24), or 2 << 24 (overflow record) when p - r
 * is not in the core.  The kernels read the same table (every point with
 * |p|^2 <= 22; farther points are always overflow records).  Lets a CPU test
 * compare the table with other encoders. */
e8q_status e8q_escape_lookup(const int8_t* coord2, int64_t n, uint32_t* out);


/* Workspace bytes e8q_project_encode needs for these matrices (>= 16). */
size_t e8q_encode_workspace_bytes(const e8q_matrix* mats /* host [n_mats] */, int32_t n_mats);

/*
 * Project + encode (Figure 2 (b), (c); abstract): for every matrix, sign
 * flip, blockwise RHT, row scale, nearest E8 point of every group, core
 * index, escape / overflow records; optionally the dequantised weights
 * (identity-STE forward, Figure 2 (b)).  One launch covers all matrices.
 *
 * mats      host array [n_mats], 1 <= n_mats <= 448.
 * args      host pointer; buffers in it are device memory.
 * Group ids: matrix m's groups are numbered from the sum of rows*cols/8 over
 *   matrices 0..m-1, row-major inside the matrix.  The call's total group
 *   count must be < 2^31.  Rows are numbered the same way for the CSR.
 * Records: written in increasing group order.  If more records than
 *   capacity are produced, the first esc_cap / ovf_cap (in group order)
 *   are written, counters hold the true totals and n_dropped the
 *   shortfall; row_ptr offsets are the true ones (they may pass the cap).
 * ws, ws_bytes: at least e8q_encode_workspace_bytes(); the call clears it.
 * Errors: E8Q_ERR_INVALID_ARG for NULL required pointers, bad shapes,
 *   block, dtype, kappa, flags or misaligned buffers; E8Q_ERR_UNSUPPORTED
 *   for cols > 16384 or too many groups; E8Q_ERR_WORKSPACE; E8Q_ERR_CUDA.
 * flags: E8Q_ENCODE_CORE_ONLY selects the core-clipped projection,
 *   E8Q_ENCODE_SHAPE_GAIN the shape-gain code (either way esc / ovf may be
 *   NULL with zero capacity; the counters and row pointers report no
 *   records); both together are INVALID_ARG.
 */
e8q_status e8q_project_encode(const e8q_matrix* mats, int32_t n_mats, const e8q_encode_args* args, void* ws,
                              size_t ws_bytes, e8q_stream stream);

/*
 * Decode / dequantise (abstract: the core encoding and sparse extension
 * keep the lattice points exactly): p = core[idx] (+ root of an escape
 * record, or the overflow record's coordinates), then
 *   basis E8Q_DEQUANT_ROTATED:  out = bf16(s_r * p), one rounding of the
 *                               exact product;
 *   basis E8Q_DEQUANT_ORIGINAL: out = bf16(d (.) H_B (s_r * p) / sqrt(B)).
 * out_bf16: [rows][cols] bf16, 16-byte aligned.  m->esc 8-byte aligned.
 * Records must be listed per row through the row pointers (as the encode
 * writes them); records outside their tile's rows are ignored.  Requires
 * that the encode call dropped no records.  Asynchronous on `stream`;
 * errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
e8q_status e8q_decode(const e8q_encoded* m /* host */, int32_t basis, void* out_bf16, e8q_stream stream);

/*
 * Workspace bytes e8q_dequant_gemv needs for this matrix and batch (an upper
 * bound valid on any device; 256 for arguments the GEMV would reject).
 * Needs no GPU.
 */
size_t e8q_gemv_workspace_bytes(const e8q_encoded* m /* host */, int32_t batch);

/*
 * Dequant-GEMV from the 2-bit form (abstract: decoding throughput of the
 * 2-bit representation):
 *   y[b][r] = sum_c w~[r][c] x[b][c],  w~ = d (.) H_B (s_r p) / sqrt(B)
 *           = s_r * sum_g < p_rg , (H_B (d (.) x_b) / sqrt(B))_g >,
 * with p_rg = core[idx] (+ the root of an escape record, or the point of an
 * overflow record).  x: [batch][cols] bf16, 16-byte aligned; y: [batch][rows]
 * bf16; 1 <= batch <= 256; m->signs required; m->esc 8-byte aligned.  ws: device memory of at least
 * e8q_gemv_workspace_bytes(m, batch) bytes, 256-byte aligned, owned by the
 * caller, overwritten.
 *
 * Escape and overflow records must be listed per row through the CSR row
 * pointers and sorted by group within each row (e8q_project_encode writes
 * them so); records outside their row are ignored and record counts are
 * clamped to esc_count / ovf_count, so malformed records give wrong values
 * but no out-of-bounds access.
 *
 * Arithmetic: the rotated activations are formed in fp32, then, for the
 * tensor-core product with the exact integer coordinates, rounded to fp16
 * after a per-row power-of-two scaling chosen from the row's largest |x| (no
 * overflow is possible); fp32 accumulation; overflow records use the fp32
 * values; bf16 output (round to nearest even).  Expected relative error
 * about 1e-4 of the output norm.  The partial sums are added in a fixed
 * order, so repeated calls give the same bits.
 * Asynchronous on `stream`; errors: INVALID_ARG, UNSUPPORTED (cols > 16384),
 * WORKSPACE, CUDA.
 */
e8q_status e8q_dequant_gemv(const e8q_encoded* m /* host */, const void* x_bf16, int32_t batch, void* y_bf16,
                            void* ws, size_t ws_bytes, e8q_stream stream);

/*
 * Workspace bytes e8q_dequant_gemm needs for this matrix and batch (exact;
 * the same on every device; 256 for arguments the GEMM would reject).
 * Needs no GPU.
 */
size_t e8q_gemm_workspace_bytes(const e8q_encoded* m /* host */, int32_t batch);

/*
 * Fused dequant-GEMM from the 2-bit form, for many activation rows at once
 * (prefill and the QAT forward; E8-QAT, abstract: decoding throughput of the
 * 2-bit representation).  The same product as e8q_dequant_gemv,
 *   y[t][r] = sum_c w~[r][c] x[t][c] = s_r * sum_g < p_rg , (H_B (d (.) x_t) / sqrt(B))_g >,
 * computed without writing the dequantised weights anywhere: the codewords
 * are decoded from the indices into the tensor cores' shared-memory operand
 * (tcgen05 MMA, fp32 accumulators in tensor memory).
 * x: [batch][cols] bf16, 16-byte aligned; y: [batch][rows] bf16;
 * 1 <= batch <= 65536 (any batch is correct; on a 4096 x 14336 matrix
 * e8q_dequant_gemv is faster at 64 rows and this call at 256); m->signs required;
 * m->esc 8-byte aligned; m->ovf 4-byte aligned, ovf_count < 2^31.
 * ws: device memory of at least e8q_gemm_workspace_bytes(m, batch) bytes,
 * 256-byte aligned, owned by the caller, overwritten.  Its first 8 bytes are
 * the call's error word: 0 after a correct call; nonzero (bit 0) if one of
 * the kernel's bounded waits gave up, in which case y is not valid.
 *
 * Records: as for e8q_dequant_gemv (CSR row pointers, sorted by group within
 * each row; malformed records give wrong values but no out-of-bounds access).
 *
 * Arithmetic: the rotated activations are formed in fp32 and rounded to fp16
 * after a per-row power-of-two scaling chosen from the row's largest |x|
 * (no overflow is possible); the integer coordinates are exact in fp16 up
 * to |P_i| = 2048, and overflow points beyond that are multiplied on CUDA
 * cores with the same fp16 activations; fp32 accumulation; bf16 output
 * (round to nearest even).  Expected relative error about 1e-4 of the output
 * norm.  The K split (and with it the order of the partial sums) depends on
 * the shapes only, so repeated calls give the same bits on any device.
 * Asynchronous on `stream`; errors: INVALID_ARG, UNSUPPORTED (cols > 16384,
 * too many tiles or overflow records), WORKSPACE, CUDA.
 */
e8q_status e8q_dequant_gemm(const e8q_encoded* m /* host */, const void* x_bf16, int32_t batch, void* y_bf16,
                            void* ws, size_t ws_bytes, e8q_stream stream);

/*
 * Identity-STE backward (E8-QAT, Figure 2 (b): the projection is trained
 * with an identity straight-through estimator): the gradient of the loss
 * with respect to the latent weights equals its gradient with respect to the
 * dequantised weights, element for element, in bf16.
 *
 * grad_dequant  [n] bf16 (device): the upstream gradient dL/dW~.
 * grad_latent   [n] bf16 (device), out: dL/dW.  It may be grad_dequant
 *               itself: the identity then needs no work, and the call
 *               returns at once without launching anything (the usual use,
 *               0 bytes moved).  Otherwise the two buffers must not overlap
 *               and the call copies the n values (2n bytes read, 2n written).
 * Both pointers 2-byte aligned; 16-byte alignment of both takes the vector
 * copy.  Asynchronous on `stream`; errors: INVALID_ARG (n < 0, NULL or
 * misaligned pointers with n > 0, partially overlapping buffers), CUDA.
 */
e8q_status e8q_ste_backward(const void* grad_dequant, void* grad_latent, int64_t n, e8q_stream stream);

/*
 * Project + encode without allocating anything: the same computation and
 * outputs as e8q_project_encode, for callers that cannot allocate device
 * memory at all -- code running where cudaMalloc is unavailable or
 * forbidden (inside a fixed memory pool, a plug-in of a host framework that
 * owns all allocations, a real-time path that must not allocate).  The paper
 * has no counterpart; this is a convenience of this library.
 *
 * The ordering scratch lives in a 2 MiB array compiled into the library
 * (a file-scope __device__ array: every GPU that loads the library holds
 * it until the process exits), so there is no ws argument.  A call needs
 * 16 + 8 * tiles bytes of it, so it fits while tiles <= (2 MiB - 16) / 8 =
 * 262,142, with tiles = sum over matrices of ceil(rows / rpt) and
 * rpt = max(1, min(64, floor(4096 / cols))) rows a tile.  The weight count
 * that fits therefore depends on the width: about 134 M weights at cols = 8,
 * 268 M at 16, 537 M at 32, 1.07 G at every power-of-two width from 64 to
 * 4096, and 262,142 rows (4.3 G weights at 16384) for widths above 4096.
 * A call that needs more returns E8Q_ERR_SCRATCH_LIMIT.  The kernel is the
 * general one (any supported shape and dtype); it clears the part of the
 * scratch it uses on `stream` before running.
 *
 * The first call on each device looks up the device address of the scratch
 * array (and uploads the constant tables); make it before any stream
 * capture.  That address, like the uploaded tables, belongs to the device's
 * primary context: after cudaDeviceReset the library's per-device state is
 * stale and must not be used (reload the library in a new process).  All
 * calls share the one array: calls that overlap on the GPU (other streams,
 * other host threads) race and must be serialised by the caller.  Other
 * arguments, outputs and errors as for e8q_project_encode.
 */
e8q_status e8q_project_encode_noalloc(const e8q_matrix* mats, int32_t n_mats, const e8q_encode_args* args,
                                      e8q_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* E8Q_H */
