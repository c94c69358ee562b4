/*
 * spectra.h -- C ABI of the B200 (sm_100a) SPECTRA outlier-split INT4 library.
 *
 * The method ("SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
 * Architecture", Dev.to abstract, abstract paragraph): every input channel
 * (column j of W[n][k]) whose fourth-moment kurtosis, taken on the column
 * scaled by its upstream normalisation gain, exceeds a threshold (3.0 in the
 * abstract) is kept bit-exact in BF16; the remaining bulk is stored as Group-32
 * 4-bit codes with one FP16 scale and one bit-packed 4-bit zero point per
 * group of 32 consecutive weights of a row.  Decoding happens in registers
 * inside the matrix-vector kernel, which also runs the dense matvec of the
 * BF16 outlier columns in the same pass (abstract: the dequantisation is
 * fused into the kernels' register pipelines).  Around the matvec: the
 * packing steps, a compacted form of the bulk, rows of a packed table
 * gathered as embeddings, the Group-32 4-bit KV cache with decode attention
 * over it, and the self-contained container the layers are stored in.
 *
 * Conventions shared by every entry point:
 *   - All pointers named *_dev or documented as "device" are CUDA device
 *     pointers (global memory of the current device) owned by the caller;
 *     the library never allocates, frees or retains them.  Host pointers are
 *     documented as such.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Work is enqueued on it.  Functions documented "synchronous"
 *     wait for their own work on `stream` before returning.
 *   - Argument checks run before any launch.  A failed check returns its
 *     status and leaves every output untouched.  Launch failures return
 *     SPECTRA_ERR_CUDA.  Faults of asynchronous work surface at the caller's
 *     next synchronisation.
 *   - Device pointers must be 16-byte aligned unless an entry states a
 *     weaker rule (SPECTRA_ERR_ALIGN otherwise).
 *   - Results are bit-identical from run to run: every reduction has a fixed
 *     order.
 *   - No exception crosses the ABI.  Library state: a per-device cache of
 *     device properties (filled on first use under a lock), per-device
 *     status flags that kernels raise and spectra_device_status reads and
 *     clears, the CRC-32 tables (built once), and the fixed scratch array of
 *     spectra_pack_plan_noalloc.  Container readers are handles the caller
 *     owns (spectra_trdc_open / spectra_trdc_close).
 *
 * Shapes: n = out_features (rows of W), k = in_features (columns), m = batch
 * rows of x.  k must be a positive multiple of 32; n >= 1.
 *
 * Packed layout ("RT32", this library's Blackwell layout; it replaces the
 * Marlin interleave named in the abstract).  N_pad = ceil(n/32)*32,
 * T = N_pad/32 row tiles, G = k/32 groups, S = ceil(G/8) super-groups,
 * O8 = ceil(n_outliers/8):
 *   codes   : 16-byte record per (tile t, group g, lane r) at byte offset
 *             ((t*G + g)*32 + r)*16; the record's little-endian u32 word w
 *             holds in nibble j (bits 4j..4j+3) the code of column
 *             32g + 8w + j of row 32t + r.  A warp (lane r = row r of the
 *             tile) reads one contiguous 512-byte segment per group.
 *   scales  : FP16 bits, element ((t*S + g/8)*32 + r)*8 + g%8; one 16-byte
 *             load gives a row its 8 scales of a super-group.
 *   zeros   : u32 word (t*S + g/8)*32 + r, nibble g%8 holds the zero point.
 *   outliers: BF16 bits, element ((t*O8 + j/8)*32 + r)*8 + j%8 holds
 *             W[32t + r][idx[j]] for outlier slot j.
 *   Padding rows, groups and outlier slots are zero.  Bulk storage is
 *   4.625 bits per weight (0.578 bytes) plus 16 bits per outlier element.
 *
 * Two forms of the bulk:
 *   masked (spectra_pack): the bulk keeps all k columns and the outlier
 *     columns are set to +0 in it before quantisation (their codes decode to
 *     exactly 0); G = k/32.
 *   compacted (spectra_pack_compact): the outlier columns are removed from
 *     the bulk, which holds the k - n_outliers other columns in ascending
 *     order, padded with all-zero columns to k_bulk = max(32, 32 *
 *     ceil((k - n_outliers)/32)); bulk_idx[p] is the column of W held by
 *     bulk column p (-1 for padding); G = k_bulk/32.  Groups of 32 are then
 *     32 consecutive *bulk* columns.  The layout above applies with k_bulk in
 *     place of k; x keeps its k columns and the kernels gather it through
 *     bulk_idx.
 */
#ifndef SPECTRA_H
#define SPECTRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPECTRA_API __attribute__((visibility("default")))
#else
#define SPECTRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPECTRA_OK = 0,
    SPECTRA_ERR_INVALID_ARG = 1,      /* null pointer, negative count, bad enum value; a
                                         gathered id outside the table (device status) */
    SPECTRA_ERR_SHAPE = 2,            /* k % 32 != 0, k < 32, n < 1, m outside [1, 32], a KV
                                         shape or length out of range, too large */
    SPECTRA_ERR_ALIGN = 3,            /* a pointer is not aligned as its entry requires */
    SPECTRA_ERR_NONFINITE = 4,        /* NaN or infinity in W, in the gain, or in appended
                                         K/V values (device status) */
    SPECTRA_ERR_RANGE = 5,            /* a group's scale (max-min)/15 overflows FP16 */
    SPECTRA_ERR_BUFFER_TOO_SMALL = 6, /* workspace smaller than the stated size */
    SPECTRA_ERR_CUDA = 7,             /* a CUDA runtime call failed */
    SPECTRA_ERR_UNSUPPORTED = 8,      /* the current device is not compute capability 10.0 */
    SPECTRA_ERR_INTERNAL = 9,         /* a kernel reported an inconsistent state */
    SPECTRA_ERR_IO = 10,              /* a container file could not be opened, read or written */
    SPECTRA_ERR_FORMAT = 11           /* a container is not TRDC, is truncated, or fails a checksum */
} spectra_status;

typedef enum { SPECTRA_F32 = 0, SPECTRA_BF16 = 1 } spectra_dtype;

/* Largest number of matvecs one spectra_gemv_batched call accepts. */
#define SPECTRA_MAX_BATCH 224

/* Largest in_features k that spectra_pack_plan_noalloc accepts. */
#define SPECTRA_NOALLOC_MAX_K 65536

/* A packed layer: a plain view of caller-owned device buffers. */
typedef struct {
    int32_t n;                   /* out_features */
    int32_t k;                   /* in_features, multiple of 32 */
    int32_t n_outliers;          /* number of BF16 outlier columns, 0..k */
    const uint8_t *codes;        /* device, RT32 code records */
    const uint16_t *scales;      /* device, FP16 bits */
    const uint32_t *zeros;       /* device, 8 zero points per word */
    const int32_t *outlier_idx;  /* device, ascending column indices [n_outliers] */
    const uint16_t *outlier_w;   /* device, BF16 bits, RT32 outlier block */
    int32_t k_bulk;              /* compacted: bulk columns; masked: 0 or k */
    const int32_t *bulk_idx;     /* device [k_bulk], 16-byte aligned, compacted
                                    only; NULL selects the masked bulk */
} spectra_layer;

/* Byte sizes of the packed buffers of one layer. */
typedef struct {
    int64_t n_pad;
    size_t codes_bytes;
    size_t scales_bytes;
    size_t zeros_bytes;
    size_t outlier_idx_bytes;
    size_t outlier_w_bytes;
    int32_t k_bulk;              /* columns of the bulk (k when masked) */
    size_t bulk_idx_bytes;       /* 0 when masked */
} spectra_sizes;

/* Human-readable name of a status value (static string, never NULL). */
SPECTRA_API const char *spectra_status_string(spectra_status s);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
SPECTRA_API int32_t spectra_version(void);

/*
 * Sizes of the packed buffers for an (n x k) layer with n_outliers outlier
 * columns (layout above).  Host only, no CUDA call.
 */
SPECTRA_API spectra_status spectra_packed_sizes(int32_t n, int32_t k, int32_t n_outliers, spectra_sizes *out);

/*
 * The same for a compacted bulk (k_bulk columns, plus the bulk column list).
 * Host only, no CUDA call.
 */
SPECTRA_API spectra_status spectra_packed_sizes_compact(int32_t n, int32_t k, int32_t n_outliers,
                                                        spectra_sizes *out);

/* Device workspace bytes that spectra_pack_plan needs for in_features k. */
SPECTRA_API size_t spectra_pack_plan_workspace_size(int32_t k);

/* Device workspace bytes that spectra_pack needs (a status word). */
SPECTRA_API size_t spectra_pack_workspace_size(void);

/*
 * Saliency split (abstract: kurtosis of each channel from the upstream
 * normalisation gain; channels above the threshold go to bit-exact storage).
 *   w        device, BF16 bits, row-major [n][k]
 *   gain     device, float [k], or NULL for g = 1
 *   tau      threshold; column j is an outlier iff kappa_j > tau (strict)
 *   kappa_out  device double [k] receiving kappa_j, or NULL
 *   idx_out  device int32 [k]; receives the ascending outlier indices
 *   n_outliers_out  HOST int32; receives |O|
 *   workspace  device, >= spectra_pack_plan_workspace_size(k) bytes
 * kappa_j is the Pearson kurtosis m4/m2^2 (population moments) of
 * a_i = W[i][j]*g_j over rows i, computed in IEEE double in the fixed order
 * sum -> mean -> (d, d^2, m2 += d^2, m4 += d^4) -> m2/n, m4/n -> m4/(m2*m2),
 * with kappa := 0 when m2 == 0; the same order as the CPU oracle, so the
 * values and the split are bit-identical to it.
 * Synchronous: returns after the split is known.  Errors: SHAPE (n < 1 or
 * k < 32 or k % 32), NONFINITE (NaN/inf in w or gain), BUFFER_TOO_SMALL.
 */
SPECTRA_API spectra_status spectra_pack_plan(const uint16_t *w, const float *gain, int32_t n, int32_t k,
                                 double tau, double *kappa_out, int32_t *idx_out,
                                 int32_t *n_outliers_out, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * spectra_pack_plan for callers that cannot allocate device memory.  The
 * paper has no counterpart to this entry point; it exists for callers that
 * must not call cudaMalloc while they plan a layer (code running under a
 * foreign allocator or a pre-carved memory pool, tools that must leave a
 * process's allocations untouched).  Same arguments, results and errors as
 * spectra_pack_plan, minus the workspace: the scratch it needs (kurtosis
 * values when kappa_out is NULL, the outlier count, an error word) lives in
 * one fixed library-owned device array of 512 KiB + 256 bytes that every GPU
 * which loads the library holds until the process exits.
 *   - k must not exceed SPECTRA_NOALLOC_MAX_K (SPECTRA_ERR_SHAPE otherwise).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents.  Calls that overlap on the GPU (issued on two streams or from
 *     two host threads for the same device) race on it: serialise them.
 *     Each call clears the words that must start at zero.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress)
 *     on the current device, so an address is never reused after a reset of
 *     the device's context moved the array.
 * Synchronous, like spectra_pack_plan.
 */
SPECTRA_API spectra_status spectra_pack_plan_noalloc(const uint16_t *w, const float *gain,
                                                     int32_t n, int32_t k, double tau,
                                                     double *kappa_out, int32_t *idx_out,
                                                     int32_t *n_outliers_out, void *stream);

/*
 * Group quantiser + packer (abstract: Group-32 4-bit microscaling with
 * bit-packed zero points; outlier channels kept bit-exact).
 *   w        device, BF16 bits [n][k]
 *   idx      device int32 [n_outliers], ascending, from spectra_pack_plan
 *   codes, scales, zeros, outlier_w   device outputs sized by
 *            spectra_packed_sizes (outlier_w may be NULL when n_outliers == 0)
 *   workspace  device, >= spectra_pack_workspace_size() bytes
 *   layer_out  HOST; filled with a view of the outputs (may be NULL)
 * Per row and group of 32 columns, over W with the outlier columns set to +0
 * and -0 read as +0: lo = min, hi = max (double); s = FP16 of (hi-lo)/15 with
 * one round-to-nearest-even step; S = (double)s; S == 0 -> zero point 0 and
 * codes 0; else z = clamp(rint(-lo/S), 0, 15), c = clamp(rint(w/S) + z, 0, 15)
 * (division in IEEE double, rint ties to even).  Bit-identical to the oracle.
 * Synchronous.  Errors: SHAPE, NONFINITE, RANGE (a scale rounds to FP16
 * infinity), INVALID_ARG (an index outside [0, k) or not ascending).
 */
SPECTRA_API spectra_status spectra_pack(const uint16_t *w, int32_t n, int32_t k, const int32_t *idx,
                            int32_t n_outliers, uint8_t *codes, uint16_t *scales,
                            uint32_t *zeros, uint16_t *outlier_w, void *workspace,
                            size_t workspace_bytes, spectra_layer *layer_out, void *stream);

/*
 * spectra_pack with a compacted bulk (abstract: the heavy-tailed coordinates
 * are decoupled into bit-exact storage and the residual bulk quantised; here
 * the outlier columns leave the 4-bit bulk instead of staying in it as
 * zeros, which saves 4.625 bits per outlier element).  Arguments as
 * spectra_pack, sized by spectra_packed_sizes_compact, plus
 *   bulk_idx  device int32 [k_bulk] output, 16-byte aligned: the column of W
 *             held by each bulk column, -1 for padding
 * The quantiser is spectra_pack's, applied to the compacted bulk: per row
 * and group of 32 consecutive bulk columns.  layer_out (HOST, may be NULL)
 * receives the view with k_bulk and bulk_idx set.  Bit-identical to the
 * oracle.  Synchronous.  Errors: as spectra_pack.
 */
SPECTRA_API spectra_status spectra_pack_compact(const uint16_t *w, int32_t n, int32_t k,
                                                const int32_t *idx, int32_t n_outliers,
                                                uint8_t *codes, uint16_t *scales, uint32_t *zeros,
                                                uint16_t *outlier_w, int32_t *bulk_idx,
                                                void *workspace, size_t workspace_bytes,
                                                spectra_layer *layer_out, void *stream);

/*
 * Inverse of the layout step, for tests: packed layer -> canonical row-major
 * arrays codes [n][kb] (one code per byte), scales [n][kb/32] (FP16 bits),
 * zeros [n][kb/32] (one zero point per byte), all device, where kb is k for
 * a masked bulk and k_bulk for a compacted one.  Asynchronous.
 */
SPECTRA_API spectra_status spectra_unpack(const spectra_layer *layer, uint8_t *codes, uint16_t *scales,
                              uint8_t *zeros, void *stream);

/*
 * Batch-1 decode matvec, the hot path:
 *   y[i] = sum_g s_ig * sum_{k in g} (c_ik - z_ig) * x[k]
 *        + sum_t W[i][idx_t] * x[idx_t]
 *   layer  HOST struct viewing device buffers
 *   x      device, BF16 bits [k]
 *   y      device, [n] of y_dtype (FP32 or BF16, round to nearest even)
 * FP32 accumulation; accepted results satisfy |y - y_ref| <=
 * 2e-3 * sum_j |w_hat_ij * x_j| + 1e-5 against the FP64 oracle.
 * Asynchronous, allocates nothing, graph-capturable.  The kernel is launched
 * with programmatic dependent launch: it may start streaming its (constant)
 * packed weights while the previous kernel on the stream is finishing, and
 * it reads x and writes y only after that kernel has completed.
 * Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_gemv(const spectra_layer *layer, const uint16_t *x, void *y,
                            spectra_dtype y_dtype, void *stream);

/*
 * Small-batch decode matmul, y[m][i] for m in [0, m_rows), 1 <= m_rows <= 32:
 *   x  device, BF16 bits [m_rows][k] row-major;  y  device [m_rows][n].
 * Same formula and tolerance as spectra_gemv per batch row.  m_rows <= 7 runs
 * on CUDA cores (m_rows accumulators per lane); 8..32 runs the tensor-core
 * path: the bulk weights are dequantised in registers to FP16 operands
 * s * (c - z) (one round-to-nearest-even rounding, relative 2^-11) against x
 * converted to FP16, the outlier columns enter as exact BF16 products, and
 * each 128-row block accumulates in FP32 in tensor memory.  The FP16
 * operands bound the inputs: an x value beyond 65504 in a bulk column, or a
 * group scale of 4368 or more, yields non-finite outputs, which the kernel
 * reports through spectra_device_status as SPECTRA_ERR_RANGE (the CUDA-core
 * path, m_rows <= 7, computes in FP32 and has no such bound).
 * Asynchronous, allocates nothing.
 */
SPECTRA_API spectra_status spectra_gemm_small(const spectra_layer *layer, const uint16_t *x, int32_t m_rows,
                                  void *y, spectra_dtype y_dtype, void *stream);

/*
 * Many independent batch-1 matvecs in ONE launch: y[i] = W_i x[i] for
 * i in [0, count), 1 <= count <= SPECTRA_MAX_BATCH, each with the formula,
 * tolerance and output type of spectra_gemv.
 *   layers  HOST array [count] of layer views (device buffers)
 *   x       HOST array [count] of device pointers, BF16 bits [layers[i].k]
 *   y       HOST array [count] of device pointers, [layers[i].n] of y_dtype
 * The matvecs run concurrently: no y[i] may overlap any x[j] or another
 * y[j].  This is the decode-step weight stream when the inputs of the
 * matrices are all available (e.g. q/k/v of one layer sharing x, or the
 * stream of a whole step whose activations are given); CTAs are issued in
 * problem order, so the weights are streamed in that order.  With count = 1
 * it runs exactly as spectra_gemv.  The host arrays
 * are read during the call only.  Asynchronous, allocates nothing,
 * graph-capturable, programmatic dependent launch as spectra_gemv.
 * Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_gemv_batched(const spectra_layer *layers,
                                                const uint16_t *const *x, void *const *y,
                                                int32_t count, spectra_dtype y_dtype,
                                                void *stream);

/*
 * A dependent sequence of batch-1 matvecs in ONE launch: y[i] = W_i x[i] for
 * i = 0, 1, ..., count - 1 in that order, where x[i] may be (or may overlap)
 * the output of any earlier matvec of the call (e.g. x[i] = y[i - 1] with
 * y_dtype SPECTRA_BF16), as in a decode step whose layers feed one another.
 * The abstract's decode runs such a step replayed as a CUDA graph; this entry
 * point removes the launch per matrix: one launch of one CTA per SM spreads
 * every matvec over all SMs, and a CTA reads x[i] only after every
 * CTA has stored its rows of y[i - 1] (a device counter, release/acquire at
 * GPU scope).  The weights keep streaming across that wait.  Same formula,
 * tolerance and output type as spectra_gemv; arrays as spectra_gemv_batched,
 * 1 <= count <= SPECTRA_MAX_BATCH.  No y[i] may overlap another y[j] or an
 * x[j] with j <= i.
 *   workspace  device, >= spectra_gemv_chain_workspace_size(layers, count)
 *              bytes, 16-byte aligned: the launch's completion counter,
 *              which the call zeroes on `stream` first (cudaMemsetAsync).
 *              Consecutive calls may share it when they run in stream order.
 * Every wait on the counter is bounded (one second of %globaltimer time); a
 * wait that gives up raises the flag that spectra_device_status reports as
 * SPECTRA_ERR_INTERNAL and the launch's outputs are invalid.  The CTAs wait
 * on one another, so all of them must be resident at once: they are when no
 * kernel of another stream occupies SMs during the call; otherwise the waits
 * give up as above.  Asynchronous, allocates nothing.
 * Errors: INVALID_ARG, SHAPE, ALIGN, BUFFER_TOO_SMALL, UNSUPPORTED, CUDA.
 */
/* Workspace bytes of spectra_gemv_chain over these layers; 0 for invalid
 * arguments. */
SPECTRA_API size_t spectra_gemv_chain_workspace_size(const spectra_layer *layers, int32_t count);
SPECTRA_API spectra_status spectra_gemv_chain(const spectra_layer *layers,
                                              const uint16_t *const *x, void *const *y,
                                              int32_t count, spectra_dtype y_dtype,
                                              void *workspace, size_t workspace_bytes,
                                              void *stream);

/*
 * spectra_gemv_chain with the matvecs grouped into stages, as a decoder
 * layer's dataflow groups them (q, k and v read the same input; so do gate
 * and up).  stage: HOST array [count], nondecreasing (the call reads it
 * during the call only); matvec i reads x[i] only after every matvec of the
 * stages before stage[i] has stored y, and the matvecs of one stage run with
 * no wait between them.  So x[i] may be (or overlap) the output of any
 * matvec of an earlier stage, never of its own stage, and no y[i] may
 * overlap another y[j] or an x[j] of the same or an earlier stage.  With
 * stage[i] = i it is spectra_gemv_chain.  Workspace, waits, limits and
 * errors as spectra_gemv_chain; a decreasing stage array is INVALID_ARG.
 */
SPECTRA_API spectra_status spectra_gemv_chain_staged(const spectra_layer *layers,
                                                     const uint16_t *const *x, void *const *y,
                                                     int32_t count, spectra_dtype y_dtype,
                                                     const int32_t *stage, void *workspace,
                                                     size_t workspace_bytes, void *stream);

/*
 * Embedding-row gather over a packed table (abstract: SpectraFusedEmbedding,
 * dequantisation of vocabulary embeddings on demand; highlight 5: vocabulary
 * tables stored in the 4-bit Group-32 format, rows gathered and dequantised
 * during the forward pass).
 *   table  HOST struct viewing a packed layer of the table E[n][k] (n =
 *          vocabulary rows, k = hidden size), packed by spectra_pack_plan +
 *          spectra_pack like any layer; a tied LM head's buffers serve as is
 *   ids    device int32 [m] row ids
 *   m      number of rows, >= 0; m == 0 returns SPECTRA_OK without touching
 *          CUDA
 *   out    device [m][k] of out_dtype, 16-byte aligned
 * out[r][j] = (c - z) * s of row ids[r] for bulk columns j (exact in FP32;
 * BF16 output rounds it once, to nearest even) and the stored BF16 value
 * W[ids[r]][j], bit for bit, for outlier columns j.  An id outside [0, n)
 * yields a zero row and raises the device flag that spectra_device_status
 * reports as SPECTRA_ERR_INVALID_ARG; nothing is read or written out of
 * bounds.  Asynchronous, allocates nothing, graph-capturable; launched with
 * programmatic dependent launch (it reads ids only after the previous kernel
 * on the stream has completed).
 * Each row is assembled in shared memory, so k * (4 for FP32, 2 for BF16)
 * must fit the device's shared memory per block (B200: k <= 58112 for FP32,
 * 116224 for BF16 rows).
 * Errors: INVALID_ARG, SHAPE (m < 0, a bad table shape, or a row too large
 * for shared memory), ALIGN, UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_embed(const spectra_layer *table, const int32_t *ids, int32_t m,
                                         void *out, spectra_dtype out_dtype, void *stream);

/*
 * Row table: the layout for a table that is only gathered (an untied
 * embedding).  The RT32 layout serves the matvec (a warp streams whole
 * 32-row tiles) and puts a row's 16-byte records 512 bytes apart, so a
 * gathered row moves whole DRAM lines for every record.  A row table keeps
 * every row's pieces contiguous, G = k_bulk/32, S = ceil(G/8):
 *   codes     : record (i*G + g)*16 bytes, the 32 codes of group g of row i
 *               (word w, nibble j = bulk column 32g + 8w + j, as in RT32);
 *   scales    : FP16 bits, element i*G + g;
 *   zeros     : u32 word i*S + g/8, nibble g%8;
 *   outlier_w : BF16 bits, element i*n_outliers + o = W[i][outlier_idx[o]];
 *   outlier_idx and bulk_idx as in the layer.
 * A row-table view is a spectra_layer whose four data buffers hold this
 * layout (no padding rows).  Pass it only to spectra_embed_rows.
 *
 * spectra_row_table_sizes: bytes of each buffer for converting `layer`
 * (n_pad = n; bulk_idx_bytes is 0 for a masked bulk).  Host only.
 * spectra_row_table_from_layer: writes the row table of packed layer
 * `layer` (RT32) into caller-owned device buffers codes (16-byte aligned),
 * scales, zeros (4-byte aligned) and outlier_w (NULL when there are no
 * outlier columns), a pure permutation of the layer's bytes, and fills
 * *table_out with a view that shares the layer's outlier_idx and bulk_idx.
 * Asynchronous, allocates nothing.
 * spectra_embed_rows: spectra_embed over a row-table view: same output, bit
 * for bit, and the same handling of bad ids; a requested row reads its
 * contiguous pieces (k_bulk/2 + k_bulk/16 + 4S + 2*n_outliers bytes).
 * Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_row_table_sizes(const spectra_layer *layer, spectra_sizes *out);
SPECTRA_API spectra_status spectra_row_table_from_layer(const spectra_layer *layer, uint8_t *codes,
                                                        uint16_t *scales, uint32_t *zeros,
                                                        uint16_t *outlier_w, spectra_layer *table_out,
                                                        void *stream);
SPECTRA_API spectra_status spectra_embed_rows(const spectra_layer *table, const int32_t *ids, int32_t m,
                                              void *out, spectra_dtype out_dtype, void *stream);

/*
 * Health of the kernels on the current device.  The matvec kernels' waits
 * for the asynchronous weight copies are bounded: a wait that gives up
 * raises a per-device flag instead of hanging, and the outputs of that
 * launch are invalid.  The embedding gather raises its own flag for an id
 * outside the table (or an outlier index outside [0, k)), and the KV append
 * for a non-finite value or an FP16 scale overflow.  Returns, for what
 * happened since the last call (and clears every flag):
 * SPECTRA_ERR_INTERNAL if a wait gave up, else SPECTRA_ERR_INVALID_ARG if the
 * gather saw a bad id, else SPECTRA_ERR_NONFINITE from the KV append, else
 * SPECTRA_ERR_RANGE from the KV append (a scale overflowing FP16) or from the
 * tensor-core matmul (an FP16 operand out of range), else SPECTRA_OK.
 * Synchronous on `stream`.
 */
SPECTRA_API spectra_status spectra_device_status(void *stream);

/*
 * Exercises the failure path of the kernels' bounded waits without a fault.
 * kind 0 launches one warp that acquires a stage of a weight ring (the
 * cp.async.bulk + mbarrier ring of the matvec kernels) that no copy ever
 * fills; kind 1 launches a thread that waits, as a CTA of spectra_gemv_chain
 * waits for the others, on a device counter that nothing increments.  The
 * wait gives up after the kernels' limit (one second of %globaltimer time),
 * the launch raises the flag that spectra_device_status then reports as
 * SPECTRA_ERR_INTERNAL, and the context stays usable.
 * For tests of callers' error handling; asynchronous, allocates nothing.
 * Errors: INVALID_ARG (unknown kind), UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_selftest_wait(int32_t kind, void *stream);

/*
 * Group-32 4-bit KV cache (abstract: microscaled Group-32 4-bit key-value
 * caching keeps long contexts resident).  Each token's vector of one KV head
 * (head_dim = D channels, D a multiple of 32, at most 256) is quantised with
 * the weight quantiser of spectra_pack: D/32 groups of 32 consecutive
 * channels, an FP16 scale and a 4-bit zero point each.  One cache holds K
 * or V.  Layout, slot = head * capacity + position, G = D/32:
 *   codes : 16-byte record per (slot, group g) at byte (slot*G + g)*16;
 *           word w, nibble j = code of channel 32g + 8w + j (a token's codes
 *           are D/2 contiguous bytes);
 *   scales: FP16 bits, element slot*G + g;
 *   zeros : u32 word slot, nibble g.
 * 4.625 bits per cached value instead of 16.
 */
typedef struct {
    int32_t n_heads;     /* KV heads */
    int32_t head_dim;    /* D */
    int32_t capacity;    /* positions per head */
    uint8_t *codes;      /* device, 16-byte aligned, n_heads*capacity*D/2 bytes */
    uint16_t *scales;    /* device, n_heads*capacity*D/32 FP16 */
    uint32_t *zeros;     /* device, n_heads*capacity words */
} spectra_kv;

/* Byte sizes of a cache's three buffers (host only, no CUDA call). */
SPECTRA_API spectra_status spectra_kv_sizes(int32_t n_heads, int32_t head_dim, int32_t capacity,
                                            size_t *codes_bytes, size_t *scales_bytes,
                                            size_t *zeros_bytes);

/*
 * Quantise n_tok new tokens into positions pos .. pos + n_tok - 1:
 *   x  device, BF16 bits [n_tok][n_heads][head_dim] (a K or V projection's
 *      output layout)
 * Bit-identical to the oracle (the weight quantiser per token and head).
 * A group holding a NaN or infinity, or whose scale overflows FP16, is
 * stored as zeros and raises the flag that spectra_device_status reports
 * (NONFINITE, RANGE).  n_tok == 0 returns SPECTRA_OK without touching CUDA.
 * Asynchronous.  Errors: INVALID_ARG, SHAPE (pos + n_tok > capacity), ALIGN,
 * UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_kv_append(const spectra_kv *cache, const uint16_t *x,
                                             int32_t n_tok, int32_t pos, void *stream);

/* Device workspace bytes that spectra_attention_decode needs. */
SPECTRA_API size_t spectra_attention_workspace_size(int32_t n_q_heads, int32_t head_dim,
                                                    int32_t length);

/*
 * Decode attention of one query token over positions 0 .. length - 1 of a
 * K and a V cache of the same geometry (grouped-query heads: query head i
 * reads KV head i / (n_q_heads / n_heads), at most 8 query heads per KV head):
 *   s_t = scale * sum_d q[i][d] * k_hat[t][d],  p = softmax(s),
 *   out[i][d] = sum_t p_t * v_hat[t][d],  x_hat = (c - z) * s dequantised
 *   in registers (exact in FP32), FP32 accumulation and softmax.
 *   q    device, BF16 bits [n_q_heads][head_dim]
 *   out  device, float [n_q_heads][head_dim]
 *   workspace  device, 16-byte aligned, >= spectra_attention_workspace_size
 * Accepted results stay within (2e-3 + expm1(4e-3 * S_max)) * sum_t p_t
 * |v_hat_td| + 1e-5 of the FP64 oracle, S_max = max_t scale * sum_d |q_d
 * k_hat_td| (the matvec's 2e-3 per dot product carried through the softmax).
 * Asynchronous, allocates nothing, deterministic.  Errors: INVALID_ARG,
 * SHAPE, ALIGN, BUFFER_TOO_SMALL, UNSUPPORTED, CUDA.
 */
SPECTRA_API spectra_status spectra_attention_decode(const spectra_kv *k, const spectra_kv *v,
                                                    const uint16_t *q, int32_t n_q_heads,
                                                    int32_t length, float scale, float *out,
                                                    void *workspace, size_t workspace_bytes,
                                                    void *stream);

/*
 * TRDC container (abstract: every weight, scale and offset is serialised
 * into one self-contained binary container that is streamed straight into
 * GPU memory, so that initialisation has a bounded memory spike).  The
 * pages give no byte format; this one is the library's own.  Little-endian
 * throughout:
 *   file header, 64 bytes:
 *     0  "TRDC"   4  u32 version (1)   8  u32 layer count L
 *     12 u32 header bytes H = 64 + 256 * L   16 u64 file bytes
 *     24 u32 CRC-32 of the L layer records   28..63 zero
 *   L layer records of 256 bytes each, from byte 64:
 *     0   name, 96 bytes, NUL-padded (at most 95 characters)
 *     96  i32 n, i32 k, i32 n_outliers, i32 k_bulk (0: masked bulk)
 *     112 f64 tau (the threshold the layer was split at; informative)
 *     120 u32 flags (bit 0: compacted bulk), u32 zero
 *     128 six (u64 offset, u64 bytes) pairs: codes, scales, zeros,
 *         outlier_idx, outlier_w, bulk_idx (bytes 0 where absent)
 *     224 six u32 CRC-32 of those buffers (0 where absent)
 *     248 u64 zero
 *   buffers at offsets that are multiples of 4096, in layer and buffer
 *   order, zero padding between them; their sizes are those of
 *   spectra_packed_sizes (masked) or spectra_packed_sizes_compact.
 * CRC-32 is the IEEE 802.3 polynomial, reflected (0xEDB88320), initial and
 * final XOR 0xFFFFFFFF (the checksum of zlib and PNG).
 *
 * Host memory: every entry streams through a caller-owned staging buffer
 * (pinned host memory for device transfers) in chunks of half its size,
 * double-buffered (the file read of one chunk overlaps the copy of the
 * other).  The library allocates no host memory proportional to the
 * model: only the reader handle (the layer records).
 * Threads: checksums of chunks of 4 MB and more are computed on up to eight
 * short-lived helper threads (and, while loading, on a thread that runs
 * beside the next file read); every thread is joined before the call
 * returns.  A reader handle may serve concurrent spectra_trdc_load calls
 * (reads use explicit offsets); spectra_trdc_close must not overlap them.
 */
typedef enum { SPECTRA_MEM_DEVICE = 0, SPECTRA_MEM_HOST = 1 } spectra_memory;

/* The 256-byte layer record of a container, as read. */
typedef struct {
    char name[96];
    int32_t n, k, n_outliers, k_bulk;
    double tau;
    uint32_t flags;
    uint64_t offset[6];
    uint64_t bytes[6];
    uint32_t crc32[6];
} spectra_trdc_layer;

/* Opaque reader handle. */
typedef struct spectra_trdc spectra_trdc;

/* CRC-32 of a host buffer (as stored in containers); `crc` is 0 to start. */
SPECTRA_API uint32_t spectra_crc32(uint32_t crc, const void *data, size_t bytes);

/*
 * Write a container of `count` packed layers.
 *   path     HOST string; the file is created or truncated
 *   names    HOST array [count] of NUL-terminated names (< 96 bytes each)
 *   layers   HOST array [count] of layer views; their buffers are device
 *            memory (mem = SPECTRA_MEM_DEVICE) or host memory
 *            (SPECTRA_MEM_HOST: no CUDA call is made)
 *   taus     HOST array [count], or NULL (stored as 0)
 *   staging  HOST buffer of staging_bytes (>= 8192, pinned for device
 *            memory); buffers move through it in chunks of half its size.
 *            Required for device memory; for host memory it may be NULL
 *            (buffers are written directly) or given (same chunked path)
 * Synchronous (device copies run on `stream`).  Errors: INVALID_ARG,
 * SHAPE, BUFFER_TOO_SMALL, IO, CUDA.
 */
SPECTRA_API spectra_status spectra_trdc_write(const char *path, int32_t count,
                                              const char *const *names,
                                              const spectra_layer *layers, const double *taus,
                                              spectra_memory mem, void *staging,
                                              size_t staging_bytes, void *stream);

/*
 * Open a container: reads and checks the header and the layer records
 * (magic, version, record checksum, every layer's shape, buffer sizes and
 * offsets within the file).  *out receives a handle to release with
 * spectra_trdc_close.  Errors: INVALID_ARG, IO, FORMAT.
 */
SPECTRA_API spectra_status spectra_trdc_open(const char *path, spectra_trdc **out);

/* Number of layers in an open container (0 for NULL). */
SPECTRA_API int32_t spectra_trdc_count(const spectra_trdc *t);

/* Record of layer i (INVALID_ARG when i is out of range). */
SPECTRA_API spectra_status spectra_trdc_info(const spectra_trdc *t, int32_t i,
                                             spectra_trdc_layer *out);

/*
 * Stream layer i into caller-allocated buffers sized by its record
 * (codes, scales, zeros; outlier_idx and outlier_w when n_outliers > 0;
 * bulk_idx when compacted; the others may be NULL), in device memory
 * (mem = SPECTRA_MEM_DEVICE, 16-byte aligned) or host memory
 * (SPECTRA_MEM_HOST: no CUDA call).  staging as for spectra_trdc_write
 * (required for device memory, optional for host memory).  verify != 0
 * checks every buffer's
 * CRC-32 while it streams (FORMAT on a mismatch).  layer_out (HOST, may be
 * NULL) receives the view of the loaded buffers.  Synchronous.  Errors:
 * INVALID_ARG, ALIGN, BUFFER_TOO_SMALL, IO, FORMAT, CUDA.
 */
SPECTRA_API spectra_status spectra_trdc_load(const spectra_trdc *t, int32_t i, uint8_t *codes,
                                             uint16_t *scales, uint32_t *zeros,
                                             int32_t *outlier_idx, uint16_t *outlier_w,
                                             int32_t *bulk_idx, spectra_memory mem,
                                             void *staging, size_t staging_bytes, int32_t verify,
                                             spectra_layer *layer_out, void *stream);

/* Release a reader handle (NULL is ignored). */
SPECTRA_API void spectra_trdc_close(spectra_trdc *t);

#ifdef __cplusplus
}
#endif

#endif /* SPECTRA_H */
