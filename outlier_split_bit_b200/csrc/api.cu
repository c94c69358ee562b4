// api.cu -- extern "C" entry points declared in spectra.h.
//
// Every entry point validates its arguments on the host before it touches
// CUDA, so argument errors return without launching anything and can be
// tested on a machine without a GPU.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "internal.cuh"
#include "spectra.h"

namespace spectra {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
bool g_dev_valid[kMaxDevices];
DeviceInfo g_dev_info[kMaxDevices];
spectra_status g_dev_status[kMaxDevices];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

spectra_status check_shape(int32_t n, int32_t k) {
    if (n < 1 || k < 32 || (k % 32) != 0) return SPECTRA_ERR_SHAPE;
    // keep every element index below 2^31 per matrix dimension product
    if ((int64_t)n * (int64_t)k > ((int64_t)1 << 40)) return SPECTRA_ERR_SHAPE;
    return SPECTRA_OK;
}

spectra_status check_layer(const spectra_layer *l) {
    if (!l) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(l->n, l->k);
    if (st != SPECTRA_OK) return st;
    if (l->n_outliers < 0 || l->n_outliers > l->k) return SPECTRA_ERR_INVALID_ARG;
    if (!l->codes || !l->scales || !l->zeros) return SPECTRA_ERR_INVALID_ARG;
    if (l->n_outliers > 0 && (!l->outlier_idx || !l->outlier_w)) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(l->codes) || !aligned16(l->scales) || !aligned16(l->zeros))
        return SPECTRA_ERR_ALIGN;
    if (l->n_outliers > 0 && (!aligned16(l->outlier_w) || !aligned4(l->outlier_idx)))
        return SPECTRA_ERR_ALIGN;
    if (l->bulk_idx) {
        if (l->k_bulk != compact_width(l->k, l->n_outliers)) return SPECTRA_ERR_INVALID_ARG;
        if (!aligned16(l->bulk_idx)) return SPECTRA_ERR_ALIGN;
    } else if (l->k_bulk != 0 && l->k_bulk != l->k) {
        return SPECTRA_ERR_INVALID_ARG;
    }
    return SPECTRA_OK;
}

void fill_sizes(int32_t n, int32_t kb, int32_t n_outliers, spectra_sizes *out) {
    const Geometry g = Geometry::of(n, kb, n_outliers);
    const int64_t np = (int64_t)g.T * 32;
    out->n_pad = np;
    out->codes_bytes = (size_t)(np * kb / 2);
    out->scales_bytes = (size_t)(np * g.S * 8 * 2);
    out->zeros_bytes = (size_t)(np * g.S * 4);
    out->outlier_idx_bytes = (size_t)n_outliers * 4;
    out->outlier_w_bytes = (size_t)(np * g.O8 * 8 * 2);
    out->k_bulk = kb;
    out->bulk_idx_bytes = 0;
}
}  // namespace

spectra_status current_device(DeviceInfo *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SPECTRA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_dev_valid[dev]) {
        DeviceInfo d = {};
        d.device = dev;
        int optin = 0;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
        d.smem_optin = (size_t)optin;
        g_dev_info[dev] = d;
        g_dev_status[dev] =
            (d.cc_major == 10 && d.cc_minor == 0) ? SPECTRA_OK : SPECTRA_ERR_UNSUPPORTED;
        g_dev_valid[dev] = true;
    }
    *out = g_dev_info[dev];
    return g_dev_status[dev];
}

}  // namespace spectra

using namespace spectra;

extern "C" {

const char *spectra_status_string(spectra_status s) {
    switch (s) {
        case SPECTRA_OK: return "ok";
        case SPECTRA_ERR_INVALID_ARG: return "invalid argument";
        case SPECTRA_ERR_SHAPE: return "unsupported shape";
        case SPECTRA_ERR_ALIGN: return "pointer not 16-byte aligned";
        case SPECTRA_ERR_NONFINITE: return "non-finite value in weights or gain";
        case SPECTRA_ERR_RANGE: return "group scale overflows FP16";
        case SPECTRA_ERR_BUFFER_TOO_SMALL: return "workspace too small";
        case SPECTRA_ERR_CUDA: return "CUDA runtime error";
        case SPECTRA_ERR_UNSUPPORTED: return "device is not compute capability 10.0";
        case SPECTRA_ERR_INTERNAL: return "internal error";
        case SPECTRA_ERR_IO: return "container file could not be opened, read or written";
        case SPECTRA_ERR_FORMAT: return "not a valid TRDC container, or a checksum failed";
    }
    return "unknown status";
}

int32_t spectra_version(void) { return 200; }

spectra_status spectra_packed_sizes(int32_t n, int32_t k, int32_t n_outliers, spectra_sizes *out) {
    if (!out) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(n, k);
    if (st != SPECTRA_OK) return st;
    if (n_outliers < 0 || n_outliers > k) return SPECTRA_ERR_INVALID_ARG;
    fill_sizes(n, k, n_outliers, out);
    return SPECTRA_OK;
}

spectra_status spectra_packed_sizes_compact(int32_t n, int32_t k, int32_t n_outliers,
                                            spectra_sizes *out) {
    if (!out) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(n, k);
    if (st != SPECTRA_OK) return st;
    if (n_outliers < 0 || n_outliers > k) return SPECTRA_ERR_INVALID_ARG;
    const int32_t kb = compact_width(k, n_outliers);
    fill_sizes(n, kb, n_outliers, out);
    out->bulk_idx_bytes = (size_t)kb * 4;
    return SPECTRA_OK;
}

size_t spectra_pack_plan_workspace_size(int32_t k) {
    if (k < 0) return 0;
    return ((size_t)k * sizeof(double) + 255u) / 256u * 256u + 256u;
}

size_t spectra_pack_workspace_size(void) { return 256u; }

spectra_status spectra_pack_plan(const uint16_t *w, const float *gain, int32_t n, int32_t k,
                                 double tau, double *kappa_out, int32_t *idx_out,
                                 int32_t *n_outliers_out, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (!w || !idx_out || !n_outliers_out || !workspace) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(n, k);
    if (st != SPECTRA_OK) return st;
    if (tau != tau) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(workspace) || !aligned4(idx_out) ||
        (gain && !aligned4(gain)) || (kappa_out && ((uintptr_t)kappa_out & 7u)))
        return SPECTRA_ERR_ALIGN;
    if (workspace_bytes < spectra_pack_plan_workspace_size(k)) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    const size_t kap_bytes = ((size_t)k * sizeof(double) + 255u) / 256u * 256u;
    double *kappa = kappa_out ? kappa_out : (double *)ws;
    int *words = (int *)(ws + kap_bytes);  // [0] error bits, [1] outlier count
    if (cudaMemsetAsync(words, 0, 2 * sizeof(int), s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_kurtosis(w, gain, n, k, kappa, words, s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_split(kappa, k, tau, idx_out, words + 1, s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    int host[2] = {0, 0};
    if (cudaMemcpyAsync(host, words, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (host[0] & kErrNonfinite) return SPECTRA_ERR_NONFINITE;
    if (host[1] < 0 || host[1] > k) return SPECTRA_ERR_INTERNAL;
    *n_outliers_out = host[1];
    return SPECTRA_OK;
}

spectra_status spectra_pack(const uint16_t *w, int32_t n, int32_t k, const int32_t *idx,
                            int32_t n_outliers, uint8_t *codes, uint16_t *scales,
                            uint32_t *zeros, uint16_t *outlier_w, void *workspace,
                            size_t workspace_bytes, spectra_layer *layer_out, void *stream) {
    if (!w || !codes || !scales || !zeros || !workspace) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(n, k);
    if (st != SPECTRA_OK) return st;
    if (n_outliers < 0 || n_outliers > k) return SPECTRA_ERR_INVALID_ARG;
    if (n_outliers > 0 && (!idx || !outlier_w)) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros) ||
        !aligned16(workspace) || (n_outliers > 0 && (!aligned16(outlier_w) || !aligned4(idx))))
        return SPECTRA_ERR_ALIGN;
    if (workspace_bytes < spectra_pack_workspace_size()) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const Geometry g = Geometry::of(n, k, n_outliers);
    int *err = (int *)workspace;
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_quantize_pack(w, g, n_outliers > 0 ? idx : nullptr, codes, scales, zeros, err, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (launch_outlier_gather(w, g, idx, outlier_w, s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    int host = 0;
    if (cudaMemcpyAsync(&host, err, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (host & kErrBadIndex) return SPECTRA_ERR_INVALID_ARG;
    if (host & kErrNonfinite) return SPECTRA_ERR_NONFINITE;
    if (host & kErrRange) return SPECTRA_ERR_RANGE;
    if (layer_out) {
        layer_out->n = n;
        layer_out->k = k;
        layer_out->n_outliers = n_outliers;
        layer_out->codes = codes;
        layer_out->scales = scales;
        layer_out->zeros = zeros;
        layer_out->outlier_idx = idx;
        layer_out->outlier_w = outlier_w;
        layer_out->k_bulk = k;
        layer_out->bulk_idx = nullptr;
    }
    return SPECTRA_OK;
}

spectra_status spectra_pack_compact(const uint16_t *w, int32_t n, int32_t k, const int32_t *idx,
                                    int32_t n_outliers, uint8_t *codes, uint16_t *scales,
                                    uint32_t *zeros, uint16_t *outlier_w, int32_t *bulk_idx,
                                    void *workspace, size_t workspace_bytes,
                                    spectra_layer *layer_out, void *stream) {
    if (!w || !codes || !scales || !zeros || !bulk_idx || !workspace)
        return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_shape(n, k);
    if (st != SPECTRA_OK) return st;
    if (n_outliers < 0 || n_outliers > k) return SPECTRA_ERR_INVALID_ARG;
    if (n_outliers > 0 && (!idx || !outlier_w)) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros) ||
        !aligned16(bulk_idx) || !aligned16(workspace) ||
        (n_outliers > 0 && (!aligned16(outlier_w) || !aligned4(idx))))
        return SPECTRA_ERR_ALIGN;
    if (workspace_bytes < spectra_pack_workspace_size()) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int kb = compact_width(k, n_outliers);
    const Geometry gb = Geometry::of(n, kb, n_outliers);
    int *err = (int *)workspace;
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_bulk_columns(n_outliers > 0 ? idx : nullptr, n_outliers, k, kb, bulk_idx, err, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (launch_quantize_pack_compact(w, k, gb, bulk_idx, codes, scales, zeros, err, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (launch_outlier_gather(w, Geometry::of(n, k, n_outliers), idx, outlier_w, s) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    int host = 0;
    if (cudaMemcpyAsync(&host, err, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (host & kErrBadIndex) return SPECTRA_ERR_INVALID_ARG;
    if (host & kErrNonfinite) return SPECTRA_ERR_NONFINITE;
    if (host & kErrRange) return SPECTRA_ERR_RANGE;
    if (layer_out) {
        layer_out->n = n;
        layer_out->k = k;
        layer_out->n_outliers = n_outliers;
        layer_out->codes = codes;
        layer_out->scales = scales;
        layer_out->zeros = zeros;
        layer_out->outlier_idx = idx;
        layer_out->outlier_w = outlier_w;
        layer_out->k_bulk = kb;
        layer_out->bulk_idx = bulk_idx;
    }
    return SPECTRA_OK;
}

spectra_status spectra_unpack(const spectra_layer *layer, uint8_t *codes, uint16_t *scales,
                              uint8_t *zeros, void *stream) {
    spectra_status st = check_layer(layer);
    if (st != SPECTRA_OK) return st;
    if (!codes || !scales || !zeros) return SPECTRA_ERR_INVALID_ARG;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    if (launch_unpack(*layer, codes, scales, zeros, (cudaStream_t)stream) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    return SPECTRA_OK;
}

static spectra_status matvec(const spectra_layer *layer, const uint16_t *x, int32_t m, void *y,
                             spectra_dtype y_dtype, void *stream) {
    spectra_status st = check_layer(layer);
    if (st != SPECTRA_OK) return st;
    if (!x || !y) return SPECTRA_ERR_INVALID_ARG;
    if (y_dtype != SPECTRA_F32 && y_dtype != SPECTRA_BF16) return SPECTRA_ERR_INVALID_ARG;
    if (m < 1 || m > 32) return SPECTRA_ERR_SHAPE;
    if (!aligned16(x)) return SPECTRA_ERR_ALIGN;
    if (y_dtype == SPECTRA_F32 ? !aligned4(y) : ((uintptr_t)y & 1u)) return SPECTRA_ERR_ALIGN;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_gemv(*layer, x, m, y, (int)y_dtype, (cudaStream_t)stream, dev);
}

spectra_status spectra_gemv(const spectra_layer *layer, const uint16_t *x, void *y,
                            spectra_dtype y_dtype, void *stream) {
    return matvec(layer, x, 1, y, y_dtype, stream);
}

spectra_status spectra_gemm_small(const spectra_layer *layer, const uint16_t *x, int32_t m_rows,
                                  void *y, spectra_dtype y_dtype, void *stream) {
    return matvec(layer, x, m_rows, y, y_dtype, stream);
}

spectra_status spectra_gemv_batched(const spectra_layer *layers, const uint16_t *const *x,
                                    void *const *y, int32_t count, spectra_dtype y_dtype,
                                    void *stream) {
    if (!layers || !x || !y) return SPECTRA_ERR_INVALID_ARG;
    if (count < 1 || count > SPECTRA_MAX_BATCH) return SPECTRA_ERR_SHAPE;
    if (y_dtype != SPECTRA_F32 && y_dtype != SPECTRA_BF16) return SPECTRA_ERR_INVALID_ARG;
    for (int32_t i = 0; i < count; ++i) {
        spectra_status st = check_layer(&layers[i]);
        if (st != SPECTRA_OK) return st;
        if (!x[i] || !y[i]) return SPECTRA_ERR_INVALID_ARG;
        if (!aligned16(x[i])) return SPECTRA_ERR_ALIGN;
        if (y_dtype == SPECTRA_F32 ? !aligned4(y[i]) : ((uintptr_t)y[i] & 1u))
            return SPECTRA_ERR_ALIGN;
    }
    DeviceInfo dev;
    spectra_status st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_gemv_batched(layers, x, y, count, (int)y_dtype, (cudaStream_t)stream, dev);
}

size_t spectra_gemv_chain_workspace_size(const spectra_layer *layers, int32_t count) {
    if (!layers || count < 1 || count > SPECTRA_MAX_BATCH) return 0;
    for (int32_t i = 0; i < count; ++i)
        if (check_shape(layers[i].n, layers[i].k) != SPECTRA_OK) return 0;
    return gemv_chain_workspace_bytes();
}

namespace {
// Arguments of the dependent-sequence entries (host-side checks only).
spectra_status check_chain(const spectra_layer *layers, const uint16_t *const *x, void *const *y,
                           int32_t count, spectra_dtype y_dtype, void *workspace,
                           size_t workspace_bytes) {
    if (!layers || !x || !y || !workspace) return SPECTRA_ERR_INVALID_ARG;
    if (count < 1 || count > SPECTRA_MAX_BATCH) return SPECTRA_ERR_SHAPE;
    if (y_dtype != SPECTRA_F32 && y_dtype != SPECTRA_BF16) return SPECTRA_ERR_INVALID_ARG;
    if (workspace_bytes < 16) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    if (!aligned16(workspace)) return SPECTRA_ERR_ALIGN;
    for (int32_t i = 0; i < count; ++i) {
        spectra_status st = check_layer(&layers[i]);
        if (st != SPECTRA_OK) return st;
        if (!x[i] || !y[i]) return SPECTRA_ERR_INVALID_ARG;
        if (!aligned16(x[i])) return SPECTRA_ERR_ALIGN;
        if (y_dtype == SPECTRA_F32 ? !aligned4(y[i]) : ((uintptr_t)y[i] & 1u))
            return SPECTRA_ERR_ALIGN;
    }
    return SPECTRA_OK;
}
}  // namespace

spectra_status spectra_gemv_chain(const spectra_layer *layers, const uint16_t *const *x,
                                  void *const *y, int32_t count, spectra_dtype y_dtype,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    spectra_status st = check_chain(layers, x, y, count, y_dtype, workspace, workspace_bytes);
    if (st != SPECTRA_OK) return st;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_gemv_chain(layers, x, y, count, (int)y_dtype, nullptr, workspace, workspace_bytes,
                             (cudaStream_t)stream, dev);
}

spectra_status spectra_gemv_chain_staged(const spectra_layer *layers, const uint16_t *const *x,
                                         void *const *y, int32_t count, spectra_dtype y_dtype,
                                         const int32_t *stage, void *workspace,
                                         size_t workspace_bytes, void *stream) {
    spectra_status st = check_chain(layers, x, y, count, y_dtype, workspace, workspace_bytes);
    if (st != SPECTRA_OK) return st;
    if (!stage) return SPECTRA_ERR_INVALID_ARG;
    for (int32_t i = 1; i < count; ++i)
        if (stage[i] < stage[i - 1]) return SPECTRA_ERR_INVALID_ARG;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_gemv_chain(layers, x, y, count, (int)y_dtype, stage, workspace, workspace_bytes,
                             (cudaStream_t)stream, dev);
}

spectra_status spectra_embed(const spectra_layer *table, const int32_t *ids, int32_t m, void *out,
                             spectra_dtype out_dtype, void *stream) {
    spectra_status st = check_layer(table);
    if (st != SPECTRA_OK) return st;
    if (out_dtype != SPECTRA_F32 && out_dtype != SPECTRA_BF16) return SPECTRA_ERR_INVALID_ARG;
    if (m < 0) return SPECTRA_ERR_SHAPE;
    if (m == 0) return SPECTRA_OK;
    if (!ids || !out) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned4(ids) || !aligned16(out)) return SPECTRA_ERR_ALIGN;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_embed(*table, ids, m, out, (int)out_dtype, false, (cudaStream_t)stream, dev);
}

spectra_status spectra_row_table_sizes(const spectra_layer *layer, spectra_sizes *out) {
    if (!out) return SPECTRA_ERR_INVALID_ARG;
    spectra_status st = check_layer(layer);
    if (st != SPECTRA_OK) return st;
    const int32_t kb = bulk_cols(*layer);
    const Geometry g = Geometry::of(layer->n, kb, layer->n_outliers);
    out->n_pad = layer->n;
    out->codes_bytes = (size_t)layer->n * g.G * 16;
    out->scales_bytes = (size_t)layer->n * g.G * 2;
    out->zeros_bytes = (size_t)layer->n * g.S * 4;
    out->outlier_idx_bytes = (size_t)layer->n_outliers * 4;
    out->outlier_w_bytes = (size_t)layer->n * layer->n_outliers * 2;
    out->k_bulk = kb;
    out->bulk_idx_bytes = layer->bulk_idx ? (size_t)kb * 4 : 0;
    return SPECTRA_OK;
}

spectra_status spectra_row_table_from_layer(const spectra_layer *layer, uint8_t *codes, uint16_t *scales,
                                            uint32_t *zeros, uint16_t *outlier_w, spectra_layer *table_out,
                                            void *stream) {
    spectra_status st = check_layer(layer);
    if (st != SPECTRA_OK) return st;
    if (!codes || !scales || !zeros || !table_out) return SPECTRA_ERR_INVALID_ARG;
    if (layer->n_outliers > 0 && !outlier_w) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(codes) || ((uintptr_t)scales & 1u) || !aligned4(zeros) ||
        (outlier_w && ((uintptr_t)outlier_w & 1u)))
        return SPECTRA_ERR_ALIGN;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    spectra_layer t = *layer;  // shape and the (shared) index lists
    t.codes = codes;
    t.scales = scales;
    t.zeros = zeros;
    t.outlier_w = layer->n_outliers > 0 ? outlier_w : nullptr;
    st = launch_row_table(*layer, t, (cudaStream_t)stream, dev);
    if (st == SPECTRA_OK) *table_out = t;
    return st;
}

spectra_status spectra_embed_rows(const spectra_layer *table, const int32_t *ids, int32_t m, void *out,
                                  spectra_dtype out_dtype, void *stream) {
    if (!table) return SPECTRA_ERR_INVALID_ARG;
    if (table->n < 1 || table->k < 32 || (table->k % 32) != 0) return SPECTRA_ERR_SHAPE;
    if (table->n_outliers < 0 || table->n_outliers > table->k) return SPECTRA_ERR_INVALID_ARG;
    if (!table->codes || !table->scales || !table->zeros) return SPECTRA_ERR_INVALID_ARG;
    if (table->n_outliers > 0 && (!table->outlier_idx || !table->outlier_w)) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(table->codes) || ((uintptr_t)table->scales & 1u) || !aligned4(table->zeros) ||
        (table->n_outliers > 0 && (((uintptr_t)table->outlier_w & 1u) || !aligned4(table->outlier_idx))))
        return SPECTRA_ERR_ALIGN;
    if (table->bulk_idx) {
        if (table->k_bulk != compact_width(table->k, table->n_outliers)) return SPECTRA_ERR_INVALID_ARG;
        if (!aligned16(table->bulk_idx)) return SPECTRA_ERR_ALIGN;
    } else if (table->k_bulk != 0 && table->k_bulk != table->k) {
        return SPECTRA_ERR_INVALID_ARG;
    }
    if (out_dtype != SPECTRA_F32 && out_dtype != SPECTRA_BF16) return SPECTRA_ERR_INVALID_ARG;
    if (m < 0) return SPECTRA_ERR_SHAPE;
    if (m == 0) return SPECTRA_OK;
    if (!ids || !out) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned4(ids) || !aligned16(out)) return SPECTRA_ERR_ALIGN;
    DeviceInfo dev;
    spectra_status st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_embed(*table, ids, m, out, (int)out_dtype, true, (cudaStream_t)stream, dev);
}

static spectra_status check_kv(const spectra_kv *c) {
    if (!c) return SPECTRA_ERR_INVALID_ARG;
    if (c->n_heads < 1 || c->capacity < 1 || c->head_dim < 32 || c->head_dim > 256 ||
        c->head_dim % 32 != 0)
        return SPECTRA_ERR_SHAPE;
    if ((int64_t)c->n_heads * c->capacity * c->head_dim > ((int64_t)1 << 40)) return SPECTRA_ERR_SHAPE;
    if (!c->codes || !c->scales || !c->zeros) return SPECTRA_ERR_INVALID_ARG;
    if (!aligned16(c->codes) || ((uintptr_t)c->scales & 1u) || !aligned4(c->zeros))
        return SPECTRA_ERR_ALIGN;
    return SPECTRA_OK;
}

spectra_status spectra_kv_sizes(int32_t n_heads, int32_t head_dim, int32_t capacity,
                                size_t *codes_bytes, size_t *scales_bytes, size_t *zeros_bytes) {
    if (!codes_bytes || !scales_bytes || !zeros_bytes) return SPECTRA_ERR_INVALID_ARG;
    if (n_heads < 1 || capacity < 1 || head_dim < 32 || head_dim > 256 || head_dim % 32 != 0)
        return SPECTRA_ERR_SHAPE;
    const int64_t slots = (int64_t)n_heads * capacity;
    if (slots * head_dim > ((int64_t)1 << 40)) return SPECTRA_ERR_SHAPE;
    *codes_bytes = (size_t)(slots * head_dim / 2);
    *scales_bytes = (size_t)(slots * (head_dim / 32) * 2);
    *zeros_bytes = (size_t)(slots * 4);
    return SPECTRA_OK;
}

spectra_status spectra_kv_append(const spectra_kv *cache, const uint16_t *x, int32_t n_tok,
                                 int32_t pos, void *stream) {
    spectra_status st = check_kv(cache);
    if (st != SPECTRA_OK) return st;
    if (n_tok < 0 || pos < 0) return SPECTRA_ERR_INVALID_ARG;
    if ((int64_t)pos + n_tok > cache->capacity) return SPECTRA_ERR_SHAPE;
    if (n_tok == 0) return SPECTRA_OK;
    if (!x) return SPECTRA_ERR_INVALID_ARG;
    if ((uintptr_t)x & 1u) return SPECTRA_ERR_ALIGN;
    if ((int64_t)n_tok * cache->n_heads > ((int64_t)1 << 30)) return SPECTRA_ERR_SHAPE;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_kv_append(*cache, x, n_tok, pos, (cudaStream_t)stream);
}

size_t spectra_attention_workspace_size(int32_t n_q_heads, int32_t head_dim, int32_t length) {
    if (n_q_heads < 1 || head_dim < 1 || length < 1) return 0;
    return attention_workspace_bytes(n_q_heads, head_dim, length);
}

spectra_status spectra_attention_decode(const spectra_kv *k, const spectra_kv *v, const uint16_t *q,
                                        int32_t n_q_heads, int32_t length, float scale, float *out,
                                        void *workspace, size_t workspace_bytes, void *stream) {
    spectra_status st = check_kv(k);
    if (st != SPECTRA_OK) return st;
    st = check_kv(v);
    if (st != SPECTRA_OK) return st;
    if (k->n_heads != v->n_heads || k->head_dim != v->head_dim || k->capacity != v->capacity)
        return SPECTRA_ERR_SHAPE;
    if (!q || !out || !workspace) return SPECTRA_ERR_INVALID_ARG;
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return SPECTRA_ERR_INVALID_ARG;
    if (n_q_heads < 1 || n_q_heads % k->n_heads != 0 ||
        n_q_heads / k->n_heads > attention_max_group())
        return SPECTRA_ERR_SHAPE;
    if (length < 1 || length > k->capacity) return SPECTRA_ERR_SHAPE;
    if (((uintptr_t)q & 1u) || !aligned4(out) || !aligned16(workspace)) return SPECTRA_ERR_ALIGN;
    if (workspace_bytes < attention_workspace_bytes(n_q_heads, k->head_dim, length))
        return SPECTRA_ERR_BUFFER_TOO_SMALL;
    DeviceInfo dev;
    st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_attention(*k, *v, q, n_q_heads, length, scale, out, workspace,
                            (cudaStream_t)stream);
}

spectra_status spectra_selftest_wait(int32_t kind, void *stream) {
    if (kind != 0 && kind != 1) return SPECTRA_ERR_INVALID_ARG;
    DeviceInfo dev;
    spectra_status st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    return launch_wait_selftest(kind, (cudaStream_t)stream);
}

spectra_status spectra_device_status(void *stream) {
    DeviceInfo dev;
    spectra_status st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    unsigned int mv_bits = 0;
    st = device_error(&mv_bits, (cudaStream_t)stream);
    if (st != SPECTRA_OK) return st;
    unsigned int embed_bits = 0, kv_bits = 0;
    st = embed_device_error(&embed_bits, (cudaStream_t)stream);
    if (st != SPECTRA_OK) return st;
    st = kv_device_error(&kv_bits, (cudaStream_t)stream);
    if (st != SPECTRA_OK) return st;
    if (mv_bits & 1u) return SPECTRA_ERR_INTERNAL;
    if (embed_bits) return SPECTRA_ERR_INVALID_ARG;
    if (kv_bits & 1u) return SPECTRA_ERR_NONFINITE;
    if ((kv_bits & 2u) || (mv_bits & 2u)) return SPECTRA_ERR_RANGE;
    return SPECTRA_OK;
}

}  // extern "C"
