// embed.cu -- rows of a packed table, dequantised on demand (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph and highlight 5
// (SpectraFusedEmbedding): vocabulary tables stay in the 4-bit Group-32
// format and the rows a forward pass needs are gathered and dequantised on
// the fly.  The table is a packed layer like any other (n = vocabulary rows,
// k = hidden columns, outlier columns kept bit-exact in BF16), so a tied
// LM head's buffers serve as the embedding table as they are.
//
// Work decomposition.  One CTA per requested row (grid-stride over the
// ids).  The row is assembled in shared memory, then written out once with
// 16-byte coalesced stores:
//   1. thread g decodes bulk group g of the row: its 16-byte code record
//      (lane r = id % 32 of tile id / 32), its FP16 scale and zero-point
//      nibble, giving (c - z) * s exact in FP32 (a 5-bit signed integer times
//      an 11-bit significand), rounded once to nearest even for BF16 output;
//      a masked bulk fills columns 32g..32g+31 (zeros at the outlier
//      columns), a compacted bulk scatters its values to the columns its
//      bulk column list names;
//   2. after a block barrier, each thread takes outlier octets: one 16-byte
//      load of the row's 8 BF16 values and their 8 column indices, written
//      into the row, so those columns come back bit for bit;
//   3. after a second barrier the row goes out, and a third barrier frees
//      the buffer for the next row.
// Each row's records lie 512 bytes apart (the RT32 layout serves the matvec,
// where a warp reads whole tiles), so a lone row moves 32-byte sectors for
// its 16-byte records; ids in one tile share sectors through L2.
//
// An id outside [0, n) yields a zero row and raises bit 0 of a device flag;
// a column index outside [0, k) (outlier list or bulk column list) is
// skipped and raises bit 1.  Neither reads or writes out of bounds.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "internal.cuh"

namespace spectra {
namespace {

constexpr int kEmbedMaxThreads = 256;
constexpr int kEmbedCtasPerSm = 8;

// bit 0: a token id outside the table; bit 1: a column index outside [0, k).
__device__ unsigned int g_embed_error;

struct EmbedArgs {
    const uint4 *codes;
    const uint16_t *scales;
    const uint32_t *zeros;
    const int32_t *oidx;
    const uint4 *outw;
    const int32_t *bidx;  // bulk column list (compacted bulk), nullptr when masked
    const int32_t *ids;
    void *out;
    int n, k, G, S, O8, n_o, m;
};

template <bool kBF16>
__device__ __forceinline__ void put(uint8_t *row, int col, float v) {
    if constexpr (kBF16)
        reinterpret_cast<__nv_bfloat16 *>(row)[col] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float *>(row)[col] = v;
}

// kRows: the table is a row table (every row's code records, scales, zero
// words and outlier values contiguous) instead of the RT32 layout.
template <bool kBF16, bool kRows>
__global__ void __launch_bounds__(kEmbedMaxThreads) embed_kernel(const EmbedArgs a) {
    extern __shared__ uint4 rowbuf[];  // one output row: k * (2 or 4) bytes
    uint8_t *row = reinterpret_cast<uint8_t *>(rowbuf);
    constexpr int kEsz = kBF16 ? 2 : 4;
    // the table is constant, but which rows are needed is known only from the
    // ids, which the previous kernel on the stream may still be writing
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int r = blockIdx.x; r < a.m; r += gridDim.x) {
        const int id = a.ids[r];
        const bool ok = id >= 0 && id < a.n;
        if (!ok && threadIdx.x == 0) atomicOr(&g_embed_error, 1u);
        const int t = ok ? (id >> 5) : 0, lane = ok ? (id & 31) : 0;
        // 1. bulk groups
        for (int g = threadIdx.x; g < a.G; g += blockDim.x) {
            float v[32];
            if (ok) {
                uint4 rec;
                float s;
                int z;
                if constexpr (kRows) {
                    // row id's pieces are contiguous: a warp reads 512 bytes of records
                    rec = a.codes[(size_t)id * a.G + g];
                    s = __half2float(__ushort_as_half(a.scales[(size_t)id * a.G + g]));
                    z = (int)((a.zeros[(size_t)id * a.S + (g >> 3)] >> (4 * (g & 7))) & 0xFu);
                } else {
                    rec = a.codes[((size_t)t * a.G + g) * 32 + lane];
                    const size_t sg = ((size_t)t * a.S + (g >> 3)) * 32 + lane;
                    s = __half2float(__ushort_as_half(a.scales[sg * 8 + (g & 7)]));
                    z = (int)((a.zeros[sg] >> (4 * (g & 7))) & 0xFu);
                }
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
            if (a.bidx == nullptr) {
                uint4 *dst = reinterpret_cast<uint4 *>(row + (size_t)32 * kEsz * g);
                if constexpr (kBF16) {
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
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                            __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
                }
            } else {
                const int4 *bc = reinterpret_cast<const int4 *>(a.bidx + 32 * g);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int4 c4 = __ldg(bc + q);
                    const int c[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (c[e] < 0) continue;  // padding column
                        if (c[e] >= a.k) {
                            atomicOr(&g_embed_error, 2u);
                            continue;
                        }
                        put<kBF16>(row, c[e], v[4 * q + e]);
                    }
                }
            }
        }
        // 2. outlier columns: in a row table the row's values are contiguous
        //    (a thread per value, coalesced); in RT32 an octet per thread
        if constexpr (kRows) {
            if (a.n_o > 0) {
                __syncthreads();
                const uint16_t *ov = reinterpret_cast<const uint16_t *>(a.outw) + (size_t)(ok ? id : 0) * a.n_o;
                // eight columns per thread at a time: every load before the first store
                for (int j0 = threadIdx.x; j0 < a.n_o; j0 += 8 * blockDim.x) {
                    int col[8];
                    uint32_t b[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + u * (int)blockDim.x;
                        col[u] = j < a.n_o ? __ldg(a.oidx + j) : -2;
                        b[u] = (ok && j < a.n_o) ? (uint32_t)ov[j] : 0u;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (col[u] == -2) continue;  // past the last slot
                        if (col[u] < 0 || col[u] >= a.k) {
                            atomicOr(&g_embed_error, 2u);
                            continue;
                        }
                        if constexpr (kBF16)
                            reinterpret_cast<uint16_t *>(row)[col[u]] = (uint16_t)b[u];
                        else
                            reinterpret_cast<uint32_t *>(row)[col[u]] = b[u] << 16;
                    }
                }
            }
        } else if (a.n_o > 0) {
            __syncthreads();
            for (int o = threadIdx.x; o < a.O8; o += blockDim.x) {
                const uint4 wv = ok ? a.outw[((size_t)t * a.O8 + o) * 32 + lane] : make_uint4(0, 0, 0, 0);
                const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = 8 * o + e;
                    if (j >= a.n_o) break;
                    const int col = __ldg(a.oidx + j);
                    if (col < 0 || col >= a.k) {
                        atomicOr(&g_embed_error, 2u);
                        continue;
                    }
                    const uint32_t b = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                    if constexpr (kBF16)
                        reinterpret_cast<uint16_t *>(row)[col] = (uint16_t)b;
                    else
                        reinterpret_cast<uint32_t *>(row)[col] = b << 16;
                }
            }
        }
        __syncthreads();
        // 3. the row, 16 bytes per thread and store
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(a.out) + (size_t)r * a.k * kEsz);
        const int nvec = a.k * kEsz / 16;
        for (int i = threadIdx.x; i < nvec; i += blockDim.x) dst[i] = rowbuf[i];
        __syncthreads();
    }
}

template <bool kBF16, bool kRows>
cudaError_t launch(const EmbedArgs &args, unsigned grid, unsigned threads, size_t smem,
                   cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, embed_kernel<kBF16, kRows>, args);
}

std::mutex g_embed_mu;
bool g_embed_ready[4][64];

// Raise the dynamic shared-memory limit of the kernel once per device.
template <bool kBF16, bool kRows>
cudaError_t prepare(const DeviceInfo &dev) {
    std::lock_guard<std::mutex> lock(g_embed_mu);
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    bool &ready = g_embed_ready[(kBF16 ? 1 : 0) + (kRows ? 2 : 0)][dev.device];
    if (ready) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(
        embed_kernel<kBF16, kRows>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dev.smem_optin);
    if (e == cudaSuccess) ready = true;
    return e;
}

// Row-table gather: a warp per requested row (grid stride over the rows by
// all warps), no shared memory and no block barriers.  Lane l decodes groups
// l, l + 32, ... (the row's records, scales and zero words are contiguous, so
// a warp reads 512 contiguous bytes of records per round) and writes each
// group's 32 values straight out: 64 (BF16) or 128 (FP32) contiguous bytes
// per lane, or, for a compacted bulk, each value to its column.  After a
// __syncwarp (which orders the warp's writes) the lanes write the outlier
// columns' stored BF16 values over their columns.
template <bool kBF16>
__global__ void __launch_bounds__(256) embed_rows_warp_kernel(const EmbedArgs a) {
    constexpr int kEsz = kBF16 ? 2 : 4;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int warps = (int)(gridDim.x * blockDim.x) >> 5;
    for (int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); r < a.m; r += warps) {
        const int id = a.ids[r];
        const bool ok = id >= 0 && id < a.n;
        if (!ok && lane == 0) atomicOr(&g_embed_error, 1u);
        uint8_t *row = reinterpret_cast<uint8_t *>(a.out) + (size_t)r * a.k * kEsz;
        // this lane's groups g = lane, lane + 32, ...: the pieces of four of
        // them are loaded before the first is decoded
        constexpr int kPre = 4;
        for (int g0 = lane; g0 < a.G; g0 += 32 * kPre) {
            uint4 recs[kPre];
            uint16_t sbits[kPre];
            uint32_t zwords[kPre];
#pragma unroll
            for (int q = 0; q < kPre; ++q) {
                const int gq = g0 + 32 * q;
                const bool in = ok && gq < a.G;
                recs[q] = in ? a.codes[(size_t)id * a.G + gq] : make_uint4(0u, 0u, 0u, 0u);
                sbits[q] = in ? a.scales[(size_t)id * a.G + gq] : (uint16_t)0;
                zwords[q] = in ? a.zeros[(size_t)id * a.S + (gq >> 3)] : 0u;
            }
#pragma unroll
            for (int q = 0; q < kPre; ++q) {
                const int g = g0 + 32 * q;
                if (g >= a.G) break;
                float v[32];
                {
                    // zero for a bad id: its pieces were loaded as zeros
                    const float s = __half2float(__ushort_as_half(sbits[q]));
                    const int z = (int)((zwords[q] >> (4 * (g & 7))) & 0xFu);
                    const uint32_t wv[4] = {recs[q].x, recs[q].y, recs[q].z, recs[q].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w)
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            v[8 * w + j] = (float)((int)((wv[w] >> (4 * j)) & 0xFu) - z) * s;
                }
                if (a.bidx == nullptr) {
                    uint4 *dst = reinterpret_cast<uint4 *>(row + (size_t)32 * kEsz * g);
                    if constexpr (kBF16) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            uint32_t p[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * qq + 2 * e]));
                                const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[8 * qq + 2 * e + 1]));
                                p[e] = lo | (hi << 16);
                            }
                            dst[qq] = make_uint4(p[0], p[1], p[2], p[3]);
                        }
                    } else {
#pragma unroll
                        for (int qq = 0; qq < 8; ++qq)
                            dst[qq] = make_uint4(__float_as_uint(v[4 * qq]), __float_as_uint(v[4 * qq + 1]),
                                                 __float_as_uint(v[4 * qq + 2]), __float_as_uint(v[4 * qq + 3]));
                    }
                } else {
                    const int4 *bc = reinterpret_cast<const int4 *>(a.bidx + 32 * g);
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq) {
                        const int4 c4 = __ldg(bc + qq);
                        const int c[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            if (c[e] < 0) continue;  // padding column
                            if (c[e] >= a.k) {
                                atomicOr(&g_embed_error, 2u);
                                continue;
                            }
                            put<kBF16>(row, c[e], v[4 * qq + e]);
                        }
                    }
                }
            }
        }
        if (a.n_o > 0) {
            __syncwarp();  // the bulk's writes of this row come first
            const uint16_t *ov = reinterpret_cast<const uint16_t *>(a.outw) + (size_t)(ok ? id : 0) * a.n_o;
            // eight columns per lane at a time: every load before the first store
            for (int j0 = lane; j0 < a.n_o; j0 += 8 * 32) {
                int col[8];
                uint32_t b[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int j = j0 + 32 * u;
                    col[u] = j < a.n_o ? __ldg(a.oidx + j) : -2;
                    b[u] = (ok && j < a.n_o) ? (uint32_t)ov[j] : 0u;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (col[u] == -2) continue;  // past the last slot
                    if (col[u] < 0 || col[u] >= a.k) {
                        atomicOr(&g_embed_error, 2u);
                        continue;
                    }
                    if constexpr (kBF16)
                        reinterpret_cast<uint16_t *>(row)[col[u]] = (uint16_t)b[u];
                    else
                        reinterpret_cast<uint32_t *>(row)[col[u]] = b[u] << 16;
                }
            }
        }
    }
}

// RT32 -> row table: a grid-stride loop over every code record, scale, zero
// word and outlier value of the table, each copied to its row-table place
// (a permutation: nothing is recomputed).
__global__ void row_table_kernel(const uint4 *__restrict__ codes, const uint16_t *__restrict__ scales,
                                 const uint32_t *__restrict__ zeros, const uint16_t *__restrict__ outw,
                                 int n, int G, int S, int n_o, uint4 *__restrict__ rcodes,
                                 uint16_t *__restrict__ rscales, uint32_t *__restrict__ rzeros,
                                 uint16_t *__restrict__ routl) {
    const int O8 = (n_o + 7) / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t e = i0; e < (int64_t)n * G; e += stride) {
        const int64_t i = e / G, g = e - i * G, t = i >> 5, r = i & 31;
        rcodes[e] = codes[(t * G + g) * 32 + r];
        rscales[e] = scales[((t * S + (g >> 3)) * 32 + r) * 8 + (g & 7)];
    }
    for (int64_t e = i0; e < (int64_t)n * S; e += stride) {
        const int64_t i = e / S, sg = e - i * S, t = i >> 5, r = i & 31;
        rzeros[e] = zeros[(t * S + sg) * 32 + r];
    }
    for (int64_t e = i0; e < (int64_t)n * n_o; e += stride) {
        const int64_t i = e / n_o, o = e - i * n_o, t = i >> 5, r = i & 31;
        routl[e] = outw[((t * O8 + (o >> 3)) * 32 + r) * 8 + (o & 7)];
    }
}

}  // namespace

spectra_status launch_embed(const spectra_layer &l, const int32_t *ids, int m, void *out,
                            int out_type, bool rows, cudaStream_t s, const DeviceInfo &dev) {
    const bool bf16 = out_type == SPECTRA_BF16;
    const size_t smem = (size_t)l.k * (bf16 ? 2 : 4);
    if (smem > dev.smem_optin) return SPECTRA_ERR_SHAPE;
    const Geometry g = Geometry::of(l.n, bulk_cols(l), l.n_outliers);
    EmbedArgs a;
    a.codes = reinterpret_cast<const uint4 *>(l.codes);
    a.scales = l.scales;
    a.zeros = l.zeros;
    a.oidx = l.outlier_idx;
    a.outw = reinterpret_cast<const uint4 *>(l.outlier_w);
    a.bidx = l.bulk_idx;
    a.ids = ids;
    a.out = out;
    a.n = l.n;
    a.k = l.k;
    a.G = g.G;
    a.S = g.S;
    a.O8 = g.O8;
    a.n_o = l.n_outliers;
    a.m = m;
    // a thread per bulk group (whole warps, at least 128 threads for the
    // outlier octets and the row store), one CTA per row up to a few CTAs
    // per SM, the rest by grid stride
    int threads = (int)cdiv(g.G, 32) * 32;
    if (threads < 128) threads = 128;
    if (threads > kEmbedMaxThreads) threads = kEmbedMaxThreads;
    const int64_t cap = (int64_t)dev.sm_count * kEmbedCtasPerSm;
    const unsigned grid = (unsigned)(m < cap ? m : cap);
    cudaError_t e;
    if (rows && m >= 4 * dev.sm_count) {
        // many rows: a warp per row, 8 warps per CTA, up to 8 CTAs per SM
        // (few rows go to a CTA per row, whose threads share a row's groups)
        int64_t blocks = cdiv(m, 8);
        const int64_t bcap = (int64_t)dev.sm_count * 8;
        if (blocks > bcap) blocks = bcap;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)blocks, 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = s;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        e = bf16 ? cudaLaunchKernelEx(&cfg, embed_rows_warp_kernel<true>, a)
                 : cudaLaunchKernelEx(&cfg, embed_rows_warp_kernel<false>, a);
    } else if (rows) {
        e = bf16 ? prepare<true, true>(dev) : prepare<false, true>(dev);
        if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
        e = bf16 ? launch<true, true>(a, grid, (unsigned)threads, smem, s)
                 : launch<false, true>(a, grid, (unsigned)threads, smem, s);
    } else {
        e = bf16 ? prepare<true, false>(dev) : prepare<false, false>(dev);
        if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
        e = bf16 ? launch<true, false>(a, grid, (unsigned)threads, smem, s)
                 : launch<false, false>(a, grid, (unsigned)threads, smem, s);
    }
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

spectra_status launch_row_table(const spectra_layer &src, const spectra_layer &dst, cudaStream_t s,
                                const DeviceInfo &dev) {
    const Geometry g = Geometry::of(src.n, bulk_cols(src), src.n_outliers);
    const int64_t work = (int64_t)src.n * g.G;
    int64_t blocks = cdiv(work, 256);
    const int64_t cap = (int64_t)dev.sm_count * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    row_table_kernel<<<(unsigned)blocks, 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(src.codes), src.scales, src.zeros, src.outlier_w, src.n, g.G, g.S,
        src.n_outliers, reinterpret_cast<uint4 *>(const_cast<uint8_t *>(dst.codes)), const_cast<uint16_t *>(dst.scales),
        const_cast<uint32_t *>(dst.zeros), const_cast<uint16_t *>(dst.outlier_w));
    return cudaGetLastError() == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
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
