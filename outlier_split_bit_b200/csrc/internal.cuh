// internal.cuh -- declarations shared by the library's translation units.
// Device-side helpers and host launchers of the sm_100a kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "spectra.h"

namespace spectra {

// Bits of the device status word written by the packing kernels.
enum : int {
    kErrNonfinite = 1,   // NaN / infinity in W or gain
    kErrRange = 2,       // a group's FP16 scale is infinite
    kErrBadIndex = 4,    // outlier index outside [0, k) or not ascending
};

struct DeviceInfo {
    int device;
    int sm_count;
    int cc_major, cc_minor;
    size_t smem_optin;   // max dynamic shared memory per block (opt-in)
};

// Cached per-device properties of the current device.  Returns
// SPECTRA_ERR_UNSUPPORTED unless the device is compute capability 10.0.
spectra_status current_device(DeviceInfo *out);

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Geometry of the RT32 layout.
struct Geometry {
    int n, k, n_o;
    int T;      // row tiles of 32
    int G;      // groups of 32 columns
    int S;      // super-groups of 8 groups
    int O8;     // outlier octets
    static Geometry of(int n, int k, int n_o) {
        Geometry g;
        g.n = n; g.k = k; g.n_o = n_o;
        g.T = (int)cdiv(n, 32);
        g.G = k / 32;
        g.S = (int)cdiv(g.G, 8);
        g.O8 = (int)cdiv(n_o, 8);
        return g;
    }
};

// Columns of a compacted bulk: the k - n_o non-outlier columns, padded to a
// multiple of 32 and to at least one group.
inline int compact_width(int k, int n_o) {
    const int nb = k - n_o;
    return nb <= 32 ? 32 : (int)cdiv(nb, 32) * 32;
}

// Columns of a layer's bulk (the geometry of its codes, scales and zeros).
inline int bulk_cols(const spectra_layer &l) { return l.bulk_idx ? l.k_bulk : l.k; }

// ---- packing (pack.cu) ----
cudaError_t launch_kurtosis(const uint16_t *w, const float *gain, int n, int k, double *kappa,
                            int *err, cudaStream_t s);
cudaError_t launch_split(const double *kappa, int k, double tau, int32_t *idx, int *count,
                         cudaStream_t s);
cudaError_t launch_quantize_pack(const uint16_t *w, const Geometry &g, const int32_t *idx,
                                 uint8_t *codes, uint16_t *scales, uint32_t *zeros, int *err,
                                 cudaStream_t s);
// Compacted bulk: the column list (validating idx) and the quantiser over
// the bulk columns; `g` is the geometry of the bulk (k_bulk columns), `k` the
// row stride of W.
cudaError_t launch_bulk_columns(const int32_t *idx, int n_o, int k, int k_bulk, int32_t *bulk_idx,
                                int *err, cudaStream_t s);
cudaError_t launch_quantize_pack_compact(const uint16_t *w, int k, const Geometry &g,
                                         const int32_t *bulk_idx, uint8_t *codes,
                                         uint16_t *scales, uint32_t *zeros, int *err,
                                         cudaStream_t s);
cudaError_t launch_outlier_gather(const uint16_t *w, const Geometry &g, const int32_t *idx,
                                  uint16_t *outlier_w, cudaStream_t s);
cudaError_t launch_unpack(const spectra_layer &l, uint8_t *codes, uint16_t *scales, uint8_t *zeros,
                          cudaStream_t s);

// ---- matvec (gemv.cu) ----
constexpr int kMaxBatch = SPECTRA_MAX_BATCH;
// Decode matvec for 1 <= m <= 32 batch rows (CUDA cores below 8 rows, the
// tensor cores from 8).
spectra_status launch_gemv(const spectra_layer &l, const uint16_t *x, int m, void *y, int ytype,
                           cudaStream_t s, const DeviceInfo &dev);
// Reads (and clears) the matvec kernels' flags: bit 0 a bounded wait for a
// weight copy gave up, bit 1 the tensor-core path produced a non-finite
// output (an FP16 operand out of range).
spectra_status device_error(unsigned int *bits, cudaStream_t s);
// A kernel whose bounded wait can never be satisfied (kind 0: the weight
// ring's mbarrier wait); it gives up after its limit and raises the flag.
spectra_status launch_wait_selftest(int kind, cudaStream_t s);
// Independent batch-1 matvecs in one launch (count <= kMaxBatch).
spectra_status launch_gemv_batched(const spectra_layer *layers, const uint16_t *const *xs,
                                   void *const *ys, int count, int ytype, cudaStream_t s,
                                   const DeviceInfo &dev);

// A dependent sequence of batch-1 matvecs in one launch (count <= kMaxBatch):
// problem i reads x only after every problem of the earlier stages has stored
// y (stage == nullptr: every problem is its own stage, so after 0..i-1).
// `ws` holds the launch's completion counter (zeroed by the call).
spectra_status launch_gemv_chain(const spectra_layer *layers, const uint16_t *const *xs,
                                 void *const *ys, int count, int ytype, const int32_t *stage,
                                 void *ws, size_t ws_bytes, cudaStream_t s, const DeviceInfo &dev);
size_t gemv_chain_workspace_bytes();

// ---- tensor-core matmul (gemm_tc.cu) ----
// y[m][n] for 8 <= m <= 32 batch rows on the tensor cores.
spectra_status launch_tc(const spectra_layer &l, const uint16_t *x, int m, void *y, int ytype,
                         cudaStream_t s, const DeviceInfo &dev);
// Reads (and clears) the tensor-core kernel's flags (bits as device_error).
spectra_status tc_device_error(unsigned int *bits, cudaStream_t s);

// ---- embedding-row gather (embed.cu) ----
// Rows ids[0..m) of a packed table, dequantised (1 <= m).
// `rows`: the view's buffers hold the row-table layout instead of RT32.
spectra_status launch_embed(const spectra_layer &l, const int32_t *ids, int m, void *out,
                            int out_type, bool rows, cudaStream_t s, const DeviceInfo &dev);
// RT32 layer `src` -> the row-table buffers named by `dst`.
spectra_status launch_row_table(const spectra_layer &src, const spectra_layer &dst, cudaStream_t s,
                                const DeviceInfo &dev);
// Reads (and clears) the gather's flag: bit 0 a token id outside the table,
// bit 1 an outlier index outside [0, k).
spectra_status embed_device_error(unsigned int *bits, cudaStream_t s);

// ---- KV cache (kv.cu) ----
spectra_status launch_kv_append(const spectra_kv &c, const uint16_t *x, int n_tok, int pos,
                                cudaStream_t s);
spectra_status launch_attention(const spectra_kv &k, const spectra_kv &v, const uint16_t *q, int Hq,
                                int T, float scale, float *out, void *ws, cudaStream_t s);
size_t attention_workspace_bytes(int Hq, int D, int T);
int attention_max_group();
// Reads (and clears) the append's flag: bit 0 non-finite value, bit 1 FP16 range.
spectra_status kv_device_error(unsigned int *bits, cudaStream_t s);

}  // namespace spectra
