// embed.cu -- rows of a packed table, dequantised on demand (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph and highlight 5
// ("SpectraFusedEmbedding"): vocabulary tables stay in the 4-bit Group-32
// format and the rows a forward pass needs are gathered and dequantised on
// the fly.  The table is a packed layer like any other (n = vocabulary rows,
// k = hidden columns, outlier columns kept bit-exact in BF16), so a tied
// LM head's buffers serve as the embedding table as they are.
//
// Work decomposition.  One CTA per requested row (grid-stride over the ids);
// thread g of the CTA decodes group g of the row: its 16-byte code record
// (lane r = id % 32 of tile id / 32, one record per group), its FP16 scale
// and its zero-point nibble, and writes the 32 values (c - z) * s -- exact in
// FP32 (a 5-bit signed integer times an 11-bit significand) -- as eight
// 16-byte FP32 stores or four 16-byte BF16 stores (one rounding to nearest
// even).  The bulk holds exact zeros at the outlier columns; after a block
// barrier the threads overwrite those columns with the stored BF16 values,
// so they come back bit for bit.  Each row's records lie 512 bytes apart
// (the RT32 layout serves the matvec, where a warp reads whole tiles), so a
// lone row moves 32-byte sectors for 16-byte records; ids in one tile share
// sectors through L2.
//
// An id outside [0, n) yields a zero row and raises bit 0 of a device flag;
// an outlier index outside [0, k) is skipped and raises bit 1.  Neither
// reads or writes out of bounds.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.cuh"

namespace spectra {
namespace {

constexpr int kEmbedMaxThreads = 256;
constexpr int kEmbedCtasPerSm = 16;

// bit 0: a token id outside the table; bit 1: an outlier index outside [0, k).
__device__ unsigned int g_embed_error;

struct EmbedArgs {
    const uint4 *codes;
    const uint16_t *scales;
    const uint32_t *zeros;
    const int32_t *oidx;
    const uint16_t *outw;
    const int32_t *ids;
    void *out;
    int n, k, G, S, O8, n_o, m;
};

template <bool kBF16>
__global__ void __launch_bounds__(kEmbedMaxThreads) embed_kernel(const EmbedArgs a) {
    // the table is constant, but which rows are needed is known only from the
    // ids, which the previous kernel on the stream may still be writing
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int r = blockIdx.x; r < a.m; r += gridDim.x) {
        const int id = a.ids[r];
        const bool ok = id >= 0 && id < a.n;
        if (!ok && threadIdx.x == 0) atomicOr(&g_embed_error, 1u);
        const int t = ok ? (id >> 5) : 0, lane = ok ? (id & 31) : 0;
        for (int g = threadIdx.x; g < a.G; g += blockDim.x) {
            float v[32];
            if (ok) {
                const uint4 rec = a.codes[((size_t)t * a.G + g) * 32 + lane];
                const size_t sg = ((size_t)t * a.S + (g >> 3)) * 32 + lane;
                const float s = __half2float(__ushort_as_half(a.scales[sg * 8 + (g & 7)]));
                const int z = (int)((a.zeros[sg] >> (4 * (g & 7))) & 0xFu);
                const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
#pragma unroll
                for (int w = 0; w < 4; ++w)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        v[8 * w + j] = (float)((int)((wv[w] >> (4 * j)) & 0xFu) - z) * s;
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            if constexpr (kBF16) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    reinterpret_cast<__nv_bfloat16 *>(a.out) + (size_t)r * a.k + 32 * g);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * q + 2 * e]));
                        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * q + 2 * e + 1]));
                        p[e] = lo | (hi << 16);
                    }
                    dst[q] = make_uint4(p[0], p[1], p[2], p[3]);
                }
            } else {
                float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) +
                                                         (size_t)r * a.k + 32 * g);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        if (a.n_o > 0) {
            // the bulk stores of this row (zeros at the outlier columns) land
            // before the outlier values replace them
            __syncthreads();
            for (int j = threadIdx.x; j < a.n_o; j += blockDim.x) {
                const int col = a.oidx[j];
                if (col < 0 || col >= a.k) {
                    atomicOr(&g_embed_error, 2u);
                    continue;
                }
                const uint16_t b =
                    ok ? a.outw[(((size_t)t * a.O8 + (j >> 3)) * 32 + lane) * 8 + (j & 7)] : 0;
                if constexpr (kBF16)
                    reinterpret_cast<uint16_t *>(a.out)[(size_t)r * a.k + col] = b;
                else
                    reinterpret_cast<uint32_t *>(a.out)[(size_t)r * a.k + col] = (uint32_t)b << 16;
            }
        }
    }
}

template <bool kBF16>
cudaError_t launch(const EmbedArgs &args, unsigned grid, unsigned threads, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, embed_kernel<kBF16>, args);
}

}  // namespace

spectra_status launch_embed(const spectra_layer &l, const int32_t *ids, int m, void *out,
                            int out_type, cudaStream_t s, const DeviceInfo &dev) {
    const Geometry g = Geometry::of(l.n, l.k, l.n_outliers);
    EmbedArgs a;
    a.codes = reinterpret_cast<const uint4 *>(l.codes);
    a.scales = l.scales;
    a.zeros = l.zeros;
    a.oidx = l.outlier_idx;
    a.outw = l.outlier_w;
    a.ids = ids;
    a.out = out;
    a.n = l.n;
    a.k = l.k;
    a.G = g.G;
    a.S = g.S;
    a.O8 = g.O8;
    a.n_o = l.n_outliers;
    a.m = m;
    // one thread per group (rounded up to whole warps), one CTA per row up to
    // a few waves of the device, the rest by grid stride
    int threads = (int)cdiv(g.G, 32) * 32;
    if (threads > kEmbedMaxThreads) threads = kEmbedMaxThreads;
    const int64_t cap = (int64_t)dev.sm_count * kEmbedCtasPerSm;
    const unsigned grid = (unsigned)(m < cap ? m : cap);
    const cudaError_t e = out_type == SPECTRA_BF16 ? launch<true>(a, grid, (unsigned)threads, s)
                                                   : launch<false>(a, grid, (unsigned)threads, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

spectra_status embed_device_error(unsigned int *bits, cudaStream_t s) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_embed_error, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    *bits = v;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_embed_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                    s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
    }
    return SPECTRA_OK;
}

}  // namespace spectra
