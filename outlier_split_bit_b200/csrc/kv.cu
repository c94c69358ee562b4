// kv.cu -- Group-32 4-bit KV cache: append and decode attention (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: microscaled Group-32
// 4-bit key-value caching keeps long contexts resident.  Every token's
// vector of one KV head (D channels) is quantised with the weight quantiser
// (quant.cuh): D/32 groups, each with an FP16 scale and a 4-bit zero point.
//
// Layout (one slot per head h and position t, slot = h * capacity + t,
// G = D / 32): codes are 16-byte records at (slot * G + g) * 16 (word w,
// nibble j = channel 32g + 8w + j), so a token's codes are D/2 contiguous
// bytes; FP16 scales at slot * G + g; zero points in the u32 word of the
// slot, nibble g.
//
// Decode attention is split over the context ("split-K"): CTA (h, c) takes
// the KV head h and the 128 positions of chunk c.
//   1. thread t decodes K of position 128c + t -- (c - z) * s, exact in FP32
//      -- against the FP32 query rows of the head's query group, staged in
//      shared memory: one score per query head (FP32 accumulation);
//   2. per query head, the chunk's maximum m and sum l of exp(s - m);
//   3. warp w takes positions 32w .. 32w + 31, lane l channels l, l + 32, ...:
//      acc += exp(s - m) * v (FP32), reduced over the warps in fixed order.
//      Each thread loads its position's V record, scales and zero word at
//      the start (the loads overlap the K pass) and parks them in shared
//      memory, so this pass reads no global memory; the buffer is reused for
//      the cross-warp reduction.
// The partials (m, l, acc[D]) of every chunk go to the workspace and a second
// kernel merges them per query head:
//   out = sum_c exp(m_c - M) acc_c / sum_c exp(m_c - M) l_c,  M = max_c m_c.
// Every order is fixed, so results repeat bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.cuh"
#include "quant.cuh"

namespace spectra {
namespace {

constexpr int kChunk = 128;      // positions per CTA (= threads per CTA)
constexpr int kMaxGroup = 8;     // query heads per KV head

// bit 0: a non-finite value was appended; bit 1: a group's scale overflowed FP16.
__device__ unsigned int g_kv_error;

__device__ __forceinline__ double bf16_to_double(uint32_t b) {
    return (double)__uint_as_float(b << 16);
}

// One thread per (token, head): its D/32 groups, one zero-point word.
__global__ void __launch_bounds__(128) kv_append_kernel(const uint16_t *__restrict__ x, int n_tok,
                                                        int H, int D, int cap, int pos,
                                                        uint4 *__restrict__ codes,
                                                        uint16_t *__restrict__ scales,
                                                        uint32_t *__restrict__ zeros) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n_tok * H) return;
    const int t = e / H, h = e - t * H;
    const int G = D / 32;
    const size_t slot = (size_t)h * cap + pos + t;
    const uint16_t *src = x + (size_t)e * D;  // x is [n_tok][H][D]
    uint32_t zw = 0;
    unsigned int flags = 0;
    for (int g = 0; g < G; ++g) {
        double v[32];
        bool bad = false;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            const uint32_t b = src[32 * g + kk];
            bad |= (b & 0x7F80u) == 0x7F80u;
            v[kk] = __dadd_rn(bf16_to_double(b), 0.0);  // -0 + +0 = +0
        }
        uint32_t rec[4] = {0u, 0u, 0u, 0u};
        unsigned short sbits = 0;
        uint32_t z = 0;
        if (bad) {
            flags |= 1u;  // the group is stored as zeros
        } else if (!quantize_group32(v, rec, &sbits, &z)) {
            flags |= 2u;
            sbits = 0;
        }
        codes[slot * G + g] = make_uint4(rec[0], rec[1], rec[2], rec[3]);
        scales[slot * G + g] = sbits;
        zw |= z << (4 * g);
    }
    zeros[slot] = zw;
    if (flags) atomicOr(&g_kv_error, flags);
}

struct AttnArgs {
    const uint4 *kc;
    const uint16_t *ks;
    const uint32_t *kz;
    const uint4 *vc;
    const uint16_t *vs;
    const uint32_t *vz;
    const uint16_t *q;  // [Hq][D] BF16
    float scale;
    int Hq, Hkv, grp, T, cap, nch;
    float *ws_ml;   // [Hq][nch][2]: m, l
    float *ws_acc;  // [Hq][nch][D]
    float *out;     // [Hq][D]
};

template <int NG>
__global__ void __launch_bounds__(kChunk) attn_partial_kernel(const AttnArgs a) {
    constexpr int D = 32 * NG;
    constexpr int kWarps = kChunk / 32;
    // V of the chunk (phase 3), later the cross-warp partial sums
    constexpr int kVStage = kChunk * (NG * 16 + NG * 2 + 4);
    constexpr int kRed = kWarps * kMaxGroup * D * 4;
    constexpr int kPool = kVStage > kRed ? kVStage : kRed;
    __shared__ __align__(16) float qs[kMaxGroup][D];
    __shared__ float sc[kMaxGroup][kChunk];
    __shared__ __align__(16) unsigned char pool[kPool];
    __shared__ float wmax[kWarps][kMaxGroup], wsum[kWarps][kMaxGroup];
    __shared__ float cm[kMaxGroup], cl[kMaxGroup];
    uint4 *vrec_s = reinterpret_cast<uint4 *>(pool);                                 // [kChunk][NG]
    uint16_t *vsc_s = reinterpret_cast<uint16_t *>(pool + kChunk * NG * 16);         // [kChunk][NG]
    uint32_t *vz_s = reinterpret_cast<uint32_t *>(pool + kChunk * (NG * 16 + NG * 2));  // [kChunk]
    float(*red)[kMaxGroup][D] = reinterpret_cast<float(*)[kMaxGroup][D]>(pool);     // [kWarps]
    const int h = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = a.grp;
    const int tok = c * kChunk + tid;
    // this position's V, loaded now, stored to shared memory after the K pass
    uint4 vr[NG];
    uint16_t vsr[NG];
    uint32_t vzr = 0;
    if (tok < a.T) {
        const size_t slot = (size_t)h * a.cap + tok;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            vr[g] = a.vc[slot * NG + g];
            vsr[g] = a.vs[slot * NG + g];
        }
        vzr = a.vz[slot];
    } else {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            vr[g] = make_uint4(0u, 0u, 0u, 0u);
            vsr[g] = 0;
        }
    }
    // query rows of the group, FP32: every load issued before the first store
    // (a load-store loop would wait out one round trip per element)
    constexpr int kQPer = kMaxGroup * D / kChunk;
    uint32_t qraw[kQPer];
    const uint16_t *qh = a.q + (size_t)h * grp * D;  // the group's rows are contiguous
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
        const int i = tid + u * kChunk;
        qraw[u] = i < grp * D ? (uint32_t)qh[i] : 0u;
    }
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
        const int i = tid + u * kChunk;
        if (i < grp * D) qs[i / D][i % D] = __uint_as_float(qraw[u] << 16);
    }
    __syncthreads();

    // 1. scores
    float s[kMaxGroup];
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi) s[gi] = 0.f;
    if (tok < a.T) {
        const size_t slot = (size_t)h * a.cap + tok;
        const uint32_t zw = a.kz[slot];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint4 rec = a.kc[slot * NG + g];
            const float sg = __half2float(__ushort_as_half(a.ks[slot * NG + g]));
            const float nzs = -(float)((zw >> (4 * g)) & 0xFu) * sg;  // -z * s, exact
            const uint32_t wv[4] = {rec.x, rec.y, rec.z, rec.w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int j4 = 0; j4 < 2; ++j4) {
                    // channels 32g + 8w + 4*j4 .. +3: (c - z) * s = fma(c, s, -z * s),
                    // exact; c as a float by the 2^23 mantissa trick
                    float kv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t code = (wv[w] >> (4 * (4 * j4 + u))) & 0xFu;
                        kv[u] = fmaf(__uint_as_float(0x4B000000u | code) - 8388608.f, sg, nzs);
                    }
                    const int d4 = (32 * g + 8 * w + 4 * j4) / 4;
#pragma unroll
                    for (int gi = 0; gi < kMaxGroup; ++gi)
                        if (gi < grp) {
                            const float4 qv = reinterpret_cast<const float4 *>(qs[gi])[d4];
                            s[gi] = fmaf(kv[0], qv.x, s[gi]);
                            s[gi] = fmaf(kv[1], qv.y, s[gi]);
                            s[gi] = fmaf(kv[2], qv.z, s[gi]);
                            s[gi] = fmaf(kv[3], qv.w, s[gi]);
                        }
                }
        }
    }
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi)
        if (gi < grp) sc[gi][tid] = tok < a.T ? s[gi] * a.scale : -INFINITY;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        vrec_s[tid * NG + g] = vr[g];
        vsc_s[tid * NG + g] = vsr[g];
    }
    vz_s[tid] = vzr;

    // 2. chunk maximum and sum per query head (warp shuffles, then the warps in order)
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi) {
        if (gi >= grp) break;
        float m = sc[gi][tid];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) wmax[warp][gi] = m;
    }
    __syncthreads();
    if (tid < grp) {
        float m = wmax[0][tid];
        for (int w = 1; w < kWarps; ++w) m = fmaxf(m, wmax[w][tid]);
        cm[tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi) {
        if (gi >= grp) break;
        const float p = tok < a.T ? expf(sc[gi][tid] - cm[gi]) : 0.f;
        sc[gi][tid] = p;
        float l = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) wsum[warp][gi] = l;
    }
    __syncthreads();
    if (tid < grp) {
        float l = 0.f;
        for (int w = 0; w < kWarps; ++w) l += wsum[w][tid];
        cl[tid] = l;
    }

    // 3. weighted sum of V: warp w, positions 32w .. 32w + 31; lane l, channels l + 32g
    float acc[kMaxGroup][NG];
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi)
#pragma unroll
        for (int g = 0; g < NG; ++g) acc[gi][g] = 0.f;
    const int w8 = lane >> 3, sh = 4 * (lane & 7);
    const int nvalid = min(32, a.T - (c * kChunk + 32 * warp));
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
        if (i >= nvalid) break;
        const int tl = 32 * warp + i;
        const uint32_t zw = vz_s[tl];
        const uint32_t *vrec = reinterpret_cast<const uint32_t *>(vrec_s + tl * NG);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint32_t word = vrec[4 * g + w8];
            const float sg = __half2float(__ushort_as_half(vsc_s[tl * NG + g]));
            const int z = (int)((zw >> (4 * g)) & 0xFu);
            const float vval = (float)((int)((word >> sh) & 0xFu) - z) * sg;
#pragma unroll
            for (int gi = 0; gi < kMaxGroup; ++gi)
                if (gi < grp) acc[gi][g] = fmaf(sc[gi][tl], vval, acc[gi][g]);
        }
    }
    // lane l holds channel 32g + 8*(l/8) + l%8 = 32g + l; the V stage is dead
    __syncthreads();
#pragma unroll
    for (int gi = 0; gi < kMaxGroup; ++gi)
        if (gi < grp)
#pragma unroll
            for (int g = 0; g < NG; ++g) red[warp][gi][32 * g + lane] = acc[gi][g];
    __syncthreads();
    for (int i = tid; i < grp * D; i += kChunk) {
        const int gi = i / D, d = i - gi * D;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][gi][d];
        const size_t qi = (size_t)(h * grp + gi) * a.nch + c;
        a.ws_acc[qi * D + d] = v;
        if (d == 0) {
            a.ws_ml[2 * qi] = cm[gi];
            a.ws_ml[2 * qi + 1] = cl[gi];
        }
    }
}

// Merge of the chunk partials, one CTA per query head.  M (the largest chunk
// maximum) and L = sum_c exp(m_c - M) l_c come from fixed-order block
// reductions; the partial sums are staged slice by slice in shared memory
// with independent 16-byte loads (one round trip per slice), and thread d
// then sums channel d over the slice's chunks in order.
constexpr int kMergeThreads = 256;
constexpr int kMergeFloats = 8192;  // one slice: 32 KB of partial sums

__device__ float block_max(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float m = red[0];
    for (int i = 1; i < nw; ++i) m = fmaxf(m, red[i]);
    __syncthreads();
    return m;
}

__device__ float block_sum(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < nw; ++i) t += red[i];
    __syncthreads();
    return t;
}

__global__ void __launch_bounds__(kMergeThreads) attn_combine_kernel(const AttnArgs a, int D) {
    __shared__ __align__(16) float buf[kMergeFloats];
    __shared__ float wt[kMergeFloats / 32];
    __shared__ float red[kMergeThreads / 32];
    const int i = blockIdx.x, tid = threadIdx.x;
    const int nch = a.nch;
    const float *ml = a.ws_ml + (size_t)i * nch * 2;
    float m = -INFINITY;
    for (int c = tid; c < nch; c += kMergeThreads) m = fmaxf(m, ml[2 * c]);
    const float M = block_max(m, red);
    float l = 0.f;
    for (int c = tid; c < nch; c += kMergeThreads) l += expf(ml[2 * c] - M) * ml[2 * c + 1];
    const float L = block_sum(l, red);
    const int per = kMergeFloats / D;  // chunks per slice
    float o = 0.f;
    for (int c0 = 0; c0 < nch; c0 += per) {
        const int nc = min(per, nch - c0);
        const float4 *src = reinterpret_cast<const float4 *>(a.ws_acc + ((size_t)i * nch + c0) * D);
        float4 *dst = reinterpret_cast<float4 *>(buf);
        const int n4 = nc * D / 4;
        int j = tid;
        for (; j + 7 * kMergeThreads < n4; j += 8 * kMergeThreads) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = src[j + u * kMergeThreads];
#pragma unroll
            for (int u = 0; u < 8; ++u) dst[j + u * kMergeThreads] = v[u];
        }
        for (; j < n4; j += kMergeThreads) dst[j] = src[j];
        for (int c = tid; c < nc; c += kMergeThreads) wt[c] = expf(ml[2 * (c0 + c)] - M);
        __syncthreads();
        if (tid < D)
            for (int c = 0; c < nc; ++c) o = fmaf(wt[c], buf[c * D + tid], o);
        __syncthreads();
    }
    if (tid < D) a.out[(size_t)i * D + tid] = o / L;
}

template <int NG>
cudaError_t launch_attn(const AttnArgs &args, cudaStream_t s) {
    attn_partial_kernel<NG><<<dim3((unsigned)args.nch, (unsigned)args.Hkv), kChunk, 0, s>>>(args);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<<<(unsigned)args.Hq, kMergeThreads, 0, s>>>(args, 32 * NG);
    return cudaGetLastError();
}

}  // namespace

// Workspace: [Hq][nch][2] chunk statistics, then (from a 16-byte boundary)
// [Hq][nch][D] partial sums.
size_t ml_floats(int Hq, int64_t nch) { return (size_t)((Hq * nch * 2 + 3) / 4 * 4); }

size_t attention_workspace_bytes(int Hq, int D, int T) {
    const int64_t nch = cdiv(T, kChunk);
    return (ml_floats(Hq, nch) + (size_t)Hq * nch * D) * sizeof(float);
}

int attention_max_group() { return kMaxGroup; }

spectra_status launch_kv_append(const spectra_kv &c, const uint16_t *x, int n_tok, int pos,
                                cudaStream_t s) {
    const int threads = n_tok * c.n_heads;
    kv_append_kernel<<<(unsigned)cdiv(threads, 128), 128, 0, s>>>(
        x, n_tok, c.n_heads, c.head_dim, c.capacity, pos, reinterpret_cast<uint4 *>(c.codes), c.scales,
        c.zeros);
    return cudaGetLastError() == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

spectra_status launch_attention(const spectra_kv &k, const spectra_kv &v, const uint16_t *q, int Hq,
                                int T, float scale, float *out, void *ws, cudaStream_t s) {
    AttnArgs a;
    a.kc = reinterpret_cast<const uint4 *>(k.codes);
    a.ks = k.scales;
    a.kz = k.zeros;
    a.vc = reinterpret_cast<const uint4 *>(v.codes);
    a.vs = v.scales;
    a.vz = v.zeros;
    a.q = q;
    a.scale = scale;
    a.Hq = Hq;
    a.Hkv = k.n_heads;
    a.grp = Hq / k.n_heads;
    a.T = T;
    a.cap = k.capacity;
    a.nch = (int)cdiv(T, kChunk);
    a.ws_ml = static_cast<float *>(ws);
    a.ws_acc = a.ws_ml + ml_floats(Hq, a.nch);
    a.out = out;
    cudaError_t e;
    switch (k.head_dim / 32) {
        case 1: e = launch_attn<1>(a, s); break;
        case 2: e = launch_attn<2>(a, s); break;
        case 3: e = launch_attn<3>(a, s); break;
        case 4: e = launch_attn<4>(a, s); break;
        case 5: e = launch_attn<5>(a, s); break;
        case 6: e = launch_attn<6>(a, s); break;
        case 7: e = launch_attn<7>(a, s); break;
        case 8: e = launch_attn<8>(a, s); break;
        default: return SPECTRA_ERR_SHAPE;
    }
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

spectra_status kv_device_error(unsigned int *bits, cudaStream_t s) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_kv_error, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    *bits = v;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_kv_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s) !=
                cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
    }
    return SPECTRA_OK;
}

}  // namespace spectra
