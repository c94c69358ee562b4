// pack.cu -- saliency split and Group-32 packing kernels (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: per-channel
// fourth-moment kurtosis taken with the upstream normalisation gain; channels
// above the threshold kept bit-exact; Group-32 4-bit bulk with a scale and a
// bit-packed zero point per group.
//
// Every floating-point step uses the explicitly rounded double intrinsics
// (__dadd_rn, __dsub_rn, __dmul_rn, __ddiv_rn), which the compiler never
// contracts into FMA, in the order documented in spectra.h, so kappa, the
// outlier set, the scales, zero points and codes are bit-identical to an IEEE
// double evaluation in that order.  These kernels run once per weight matrix
// (offline); they favour that exact order over parallel reductions.
#include <cuda_fp16.h>

#include "internal.cuh"
#include "quant.cuh"

namespace spectra {
namespace {

__device__ __forceinline__ double bf16_to_double(uint32_t b) {
    return (double)__uint_as_float(b << 16);
}

__device__ __forceinline__ bool bf16_nonfinite(uint32_t b) { return (b & 0x7F80u) == 0x7F80u; }

// One thread per column j; rows walked in ascending order, twice.
__global__ void __launch_bounds__(128) kurtosis_kernel(const uint16_t *__restrict__ w,
                                                       const float *__restrict__ gain, int n,
                                                       int k, double *__restrict__ kappa,
                                                       int *__restrict__ err) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= k) return;
    bool bad = false;
    double g = 1.0;
    if (gain) {
        const float gf = gain[j];
        bad = !isfinite(gf);
        g = (double)gf;
    }
    const uint16_t *col = w + j;
    double s = 0.0;
#pragma unroll 8
    for (int i = 0; i < n; ++i) {
        const uint32_t b = col[(size_t)i * k];
        bad |= bf16_nonfinite(b);
        s = __dadd_rn(s, __dmul_rn(bf16_to_double(b), g));
    }
    const double mu = __ddiv_rn(s, (double)n);
    double m2 = 0.0, m4 = 0.0;
#pragma unroll 8
    for (int i = 0; i < n; ++i) {
        const double a = __dmul_rn(bf16_to_double(col[(size_t)i * k]), g);
        const double d = __dsub_rn(a, mu);
        const double q = __dmul_rn(d, d);
        m2 = __dadd_rn(m2, q);
        m4 = __dadd_rn(m4, __dmul_rn(q, q));
    }
    m2 = __ddiv_rn(m2, (double)n);
    m4 = __ddiv_rn(m4, (double)n);
    kappa[j] = (m2 == 0.0) ? 0.0 : __ddiv_rn(m4, __dmul_rn(m2, m2));
    if (bad) atomicOr(err, kErrNonfinite);
}

// Stream compaction of {j : kappa_j > tau} in ascending order; one CTA.
__global__ void __launch_bounds__(1024) split_kernel(const double *__restrict__ kappa, int k,
                                                     double tau, int32_t *__restrict__ idx,
                                                     int *__restrict__ count) {
    __shared__ int warp_off[32];
    __shared__ int chunk_total;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int base = 0;
    for (int j0 = 0; j0 < k; j0 += 1024) {
        const int j = j0 + threadIdx.x;
        const bool f = j < k && kappa[j] > tau;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const int pre = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) warp_off[warp] = __popc(bal);
        __syncthreads();
        if (warp == 0) {
            const int v = warp_off[lane];
            int incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += o;
            }
            warp_off[lane] = incl - v;
            if (lane == 31) chunk_total = incl;
        }
        __syncthreads();
        if (f) idx[base + warp_off[warp] + pre] = j;
        base += chunk_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) *count = base;
}

// Column list of a compacted bulk, one thread per column j of W: a
// non-outlier column j is bulk column j - (number of outliers below j), found
// by binary search in the ascending outlier list; positions from k - n_o to
// k_bulk are padding (-1).  Threads j < n_o also check that the list is
// strictly ascending within [0, k).  A bad list only ever writes inside
// [0, k_bulk) and is reported through err.
__global__ void __launch_bounds__(256) bulk_columns_kernel(const int32_t *__restrict__ idx,
                                                           int n_o, int k, int k_bulk,
                                                           int32_t *__restrict__ bulk_idx,
                                                           int *__restrict__ err) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j < n_o) {
        const int c = idx[j];
        if (c < 0 || c >= k || (j > 0 && idx[j - 1] >= c)) atomicOr(err, kErrBadIndex);
    }
    if (j < k) {
        int lo = 0, hi = n_o;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (idx[mid] < j)
                lo = mid + 1;
            else
                hi = mid;
        }
        const bool outlier = lo < n_o && idx[lo] == j;
        const int p = j - lo;
        if (!outlier && p >= 0 && p < k_bulk) bulk_idx[p] = j;
    }
    if (j >= k - n_o && j < k_bulk) bulk_idx[j] = -1;
}

// One thread per (tile t, super-group sg, lane r): quantises the 8 groups of
// row 32t + r in that super-group and writes its 8 code records, one 16-byte
// scale vector and one zero-point word.  Masked bulk (kCompact false): `cols`
// is the outlier list, whose columns read as +0.  Compacted bulk: `cols` is
// the bulk column list, bulk column p of the row reads W[row][cols[p]] (+0
// for padding); G and S count bulk groups and k is the row stride of W.
template <bool kCompact>
__global__ void __launch_bounds__(128) quantize_pack_kernel(
    const uint16_t *__restrict__ w, int n, int k, int T, int G, int S,
    const int32_t *__restrict__ cols, int n_o, uint4 *__restrict__ codes,
    uint4 *__restrict__ scales, uint32_t *__restrict__ zeros, int *__restrict__ err) {
    extern __shared__ uint32_t omask[];  // masked: k bits, the outlier columns
    if constexpr (!kCompact) {
        const int words = k / 32;
        for (int i = threadIdx.x; i < words; i += blockDim.x) omask[i] = 0u;
        __syncthreads();
        bool bad_idx = false;
        for (int i = threadIdx.x; i < n_o; i += blockDim.x) {
            const int j = cols[i];
            if (j < 0 || j >= k || (i > 0 && cols[i - 1] >= j)) {
                bad_idx = true;
            } else {
                atomicOr(&omask[j >> 5], 1u << (j & 31));
            }
        }
        __syncthreads();
        if (bad_idx) atomicOr(err, kErrBadIndex);
    }

    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (t, sg) pair
    const int r = threadIdx.x & 31;
    if (gw >= T * S) return;
    const int t = gw / S, sg = gw % S;
    const int row = 32 * t + r;
    int flags = 0;
    uint32_t zw = 0;
    uint32_t sc[4] = {0u, 0u, 0u, 0u};
    for (int gg = 0; gg < 8; ++gg) {
        const int g = 8 * sg + gg;
        if (g >= G) break;
        uint32_t rec[4] = {0u, 0u, 0u, 0u};
        if (row < n) {
            double v[32];
            if constexpr (kCompact) {
                const int32_t *bc = cols + 32 * g;
#pragma unroll
                for (int kk = 0; kk < 32; ++kk) {
                    const int c = bc[kk];
                    const uint32_t b = (c >= 0 && c < k) ? (uint32_t)w[(size_t)row * k + c] : 0u;
                    if (bf16_nonfinite(b)) flags |= kErrNonfinite;
                    v[kk] = __dadd_rn(bf16_to_double(b), 0.0);  // -0 + +0 = +0
                }
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(w + (size_t)row * k + 32 * g);
                uint32_t raw[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 u = src[q];
                    raw[4 * q + 0] = u.x; raw[4 * q + 1] = u.y;
                    raw[4 * q + 2] = u.z; raw[4 * q + 3] = u.w;
                }
                const uint32_t m = omask[g];
#pragma unroll
                for (int kk = 0; kk < 32; ++kk) {
                    const uint32_t b = (kk & 1) ? (raw[kk >> 1] >> 16) : (raw[kk >> 1] & 0xFFFFu);
                    if (bf16_nonfinite(b)) flags |= kErrNonfinite;
                    const double x = ((m >> kk) & 1u) ? 0.0 : bf16_to_double(b);
                    v[kk] = __dadd_rn(x, 0.0);  // -0 + +0 = +0
                }
            }
            unsigned short hbits;
            uint32_t z = 0;
            if (!quantize_group32(v, rec, &hbits, &z, (flags & kErrRange) != 0)) flags |= kErrRange;
            sc[gg >> 1] |= (uint32_t)hbits << (16 * (gg & 1));
            zw |= z << (4 * gg);
        }
        codes[((size_t)t * G + g) * 32 + r] = make_uint4(rec[0], rec[1], rec[2], rec[3]);
    }
    scales[((size_t)t * S + sg) * 32 + r] = make_uint4(sc[0], sc[1], sc[2], sc[3]);
    zeros[((size_t)t * S + sg) * 32 + r] = zw;
    if (flags) atomicOr(err, flags);
}

// One thread per (tile t, octet oc, lane r): 8 BF16 outlier weights of row
// 32t + r as one 16-byte vector.
__global__ void __launch_bounds__(128) outlier_gather_kernel(
    const uint16_t *__restrict__ w, int n, int k, int T, int O8, const int32_t *__restrict__ idx,
    int n_o, uint4 *__restrict__ outw) {
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int r = threadIdx.x & 31;
    if (gw >= T * O8) return;
    const int t = gw / O8, oc = gw % O8;
    const int row = 32 * t + r;
    uint32_t v[4] = {0u, 0u, 0u, 0u};
    if (row < n) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = 8 * oc + e;
            if (j < n_o) {
                const int col = idx[j];
                if (col >= 0 && col < k)
                    v[e >> 1] |= (uint32_t)w[(size_t)row * k + col] << (16 * (e & 1));
            }
        }
    }
    outw[((size_t)t * O8 + oc) * 32 + r] = make_uint4(v[0], v[1], v[2], v[3]);
}

// One thread per (row, group): packed -> canonical.
__global__ void __launch_bounds__(128) unpack_kernel(const uint4 *__restrict__ pcodes,
                                                     const uint16_t *__restrict__ pscales,
                                                     const uint32_t *__restrict__ pzeros, int n,
                                                     int k, int G, int S,
                                                     uint8_t *__restrict__ codes,
                                                     uint16_t *__restrict__ scales,
                                                     uint8_t *__restrict__ zeros) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)n * G) return;
    const int row = (int)(e / G), g = (int)(e % G);
    const int t = row >> 5, r = row & 31;
    const uint4 rec = pcodes[((size_t)t * G + g) * 32 + r];
    const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
    uint8_t *dst = codes + (size_t)row * k + 32 * g;
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) dst[kk] = (uint8_t)((wv[kk >> 3] >> (4 * (kk & 7))) & 0xFu);
    scales[(size_t)row * G + g] = pscales[(((size_t)t * S + g / 8) * 32 + r) * 8 + (g & 7)];
    zeros[(size_t)row * G + g] =
        (uint8_t)((pzeros[((size_t)t * S + g / 8) * 32 + r] >> (4 * (g & 7))) & 0xFu);
}

}  // namespace

cudaError_t launch_kurtosis(const uint16_t *w, const float *gain, int n, int k, double *kappa,
                            int *err, cudaStream_t s) {
    kurtosis_kernel<<<(unsigned)cdiv(k, 128), 128, 0, s>>>(w, gain, n, k, kappa, err);
    return cudaGetLastError();
}

cudaError_t launch_split(const double *kappa, int k, double tau, int32_t *idx, int *count,
                         cudaStream_t s) {
    split_kernel<<<1, 1024, 0, s>>>(kappa, k, tau, idx, count);
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack(const uint16_t *w, const Geometry &g, const int32_t *idx,
                                 uint8_t *codes, uint16_t *scales, uint32_t *zeros, int *err,
                                 cudaStream_t s) {
    const int64_t threads = (int64_t)g.T * g.S * 32;
    const size_t smem = (size_t)(g.k / 32) * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(quantize_pack_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    quantize_pack_kernel<false><<<(unsigned)cdiv(threads, 128), 128, smem, s>>>(
        w, g.n, g.k, g.T, g.G, g.S, idx, g.n_o, reinterpret_cast<uint4 *>(codes),
        reinterpret_cast<uint4 *>(scales), zeros, err);
    return cudaGetLastError();
}

cudaError_t launch_bulk_columns(const int32_t *idx, int n_o, int k, int k_bulk, int32_t *bulk_idx,
                                int *err, cudaStream_t s) {
    bulk_columns_kernel<<<(unsigned)cdiv(k, 256), 256, 0, s>>>(idx, n_o, k, k_bulk, bulk_idx, err);
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack_compact(const uint16_t *w, int k, const Geometry &g,
                                         const int32_t *bulk_idx, uint8_t *codes,
                                         uint16_t *scales, uint32_t *zeros, int *err,
                                         cudaStream_t s) {
    const int64_t threads = (int64_t)g.T * g.S * 32;
    quantize_pack_kernel<true><<<(unsigned)cdiv(threads, 128), 128, 0, s>>>(
        w, g.n, k, g.T, g.G, g.S, bulk_idx, 0, reinterpret_cast<uint4 *>(codes),
        reinterpret_cast<uint4 *>(scales), zeros, err);
    return cudaGetLastError();
}

cudaError_t launch_outlier_gather(const uint16_t *w, const Geometry &g, const int32_t *idx,
                                  uint16_t *outlier_w, cudaStream_t s) {
    if (g.O8 == 0) return cudaSuccess;
    const int64_t threads = (int64_t)g.T * g.O8 * 32;
    outlier_gather_kernel<<<(unsigned)cdiv(threads, 128), 128, 0, s>>>(
        w, g.n, g.k, g.T, g.O8, idx, g.n_o, reinterpret_cast<uint4 *>(outlier_w));
    return cudaGetLastError();
}

cudaError_t launch_unpack(const spectra_layer &l, uint8_t *codes, uint16_t *scales, uint8_t *zeros,
                          cudaStream_t s) {
    const Geometry g = Geometry::of(l.n, bulk_cols(l), l.n_outliers);
    const int64_t threads = (int64_t)l.n * g.G;
    unpack_kernel<<<(unsigned)cdiv(threads, 128), 128, 0, s>>>(
        reinterpret_cast<const uint4 *>(l.codes), l.scales, l.zeros, l.n, g.k, g.G, g.S, codes,
        scales, zeros);
    return cudaGetLastError();
}

}  // namespace spectra
