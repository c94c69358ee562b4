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
// the KV head h and the 128 positions of chunk c, with 512 threads.
//   1. four threads per position decode K -- (c - z) * s, exact in FP32 --
//      word q of every group (channels 32g + 8q .. +7), dot them with the FP32
//      query rows of the head's query group staged in shared memory, and add
//      their four partial scores with two shuffles (FP32 accumulation);
//   2. per query head, the chunk's maximum m and sum l of exp(s - m);
//   3. warp w takes positions 8w .. 8w + 7, lane l channels l, l + 32, ...:
//      acc += exp(s - m) * v (FP32), reduced over the 16 warps in fixed order.
//      Each position's V record, scales and zero word are loaded during the K
//      pass (each of the four threads one word of every group) and parked in
//      shared memory, so this pass reads no global memory.
// The partials (m, l, acc[D]) of every chunk go to the workspace and a second
// kernel, launched as a programmatic dependent of the first (its launch
// overlaps the chunks), merges them per query head and slice of 32 channels:
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

constexpr int kQuarter = 4;                        // threads per position in the K pass
constexpr int kAttnThreads = kChunk * kQuarter;    // 512
constexpr int kAttnWarps = kAttnThreads / 32;      // 16
constexpr int kStatWarps = kChunk / 32;            // warps over the chunk's positions (stats)

// Dynamic shared memory of the chunk kernel: query rows, scores, then a pool
// holding first the chunk's V records and then the cross-warp partial sums.
__host__ __device__ constexpr size_t attn_pool_bytes(int NG, int grp) {
    const size_t vstage = (size_t)kChunk * (NG * 16 + NG * 2 + 4);
    const size_t red = (size_t)kAttnWarps * grp * 32 * NG * 4;
    return vstage > red ? vstage : red;
}
__host__ __device__ constexpr size_t attn_smem_bytes(int NG, int grp) {
    return (size_t)kMaxGroup * 32 * NG * 4 + (size_t)kMaxGroup * kChunk * 4 + attn_pool_bytes(NG, grp);
}

__device__ __forceinline__ void attn_pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void attn_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// GRP: the query-group size bucket (2, 4 or 8) the registers are sized for;
// the loops run to the actual group size a.grp <= GRP.
template <int NG, int GRP>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(const AttnArgs a) {
    constexpr int D = 32 * NG;
    extern __shared__ __align__(16) unsigned char dsm[];
    float(*qs)[D] = reinterpret_cast<float(*)[D]>(dsm);                                      // [kMaxGroup][D]
    float(*sc)[kChunk] = reinterpret_cast<float(*)[kChunk]>(dsm + kMaxGroup * D * 4);          // [kMaxGroup][kChunk]
    unsigned char *pool = dsm + kMaxGroup * D * 4 + kMaxGroup * kChunk * 4;
    uint32_t *vrec_s = reinterpret_cast<uint32_t *>(pool);                                   // [kChunk][NG][4]
    uint16_t *vsc_s = reinterpret_cast<uint16_t *>(pool + kChunk * NG * 16);                 // [kChunk][NG]
    uint32_t *vz_s = reinterpret_cast<uint32_t *>(pool + kChunk * (NG * 16 + NG * 2));       // [kChunk]
    float *red = reinterpret_cast<float *>(pool);                                            // [kAttnWarps][grp][D]
    __shared__ float wmax[kStatWarps][kMaxGroup], wsum[kStatWarps][kMaxGroup];
    __shared__ float cm[kMaxGroup], cl[kMaxGroup];
    const int h = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pos = tid >> 2, qd = tid & 3;  // position in the chunk, word of each group
    const int grp = a.grp;
    const int tok = c * kChunk + pos;
    attn_pdl_launch_dependents();
    attn_pdl_wait();  // the cache and the query may come from the previous kernel
    // this position's V word qd of every group (and, thread 0 of the four,
    // the scales and zero word), parked in shared memory after the K pass
    uint32_t vw[NG];
    uint16_t vsr[NG];
    uint32_t vzr = 0;
    const size_t slot = (size_t)h * a.cap + tok;
    const bool valid = tok < a.T;
    const uint32_t *vc32 = reinterpret_cast<const uint32_t *>(a.vc);
    const uint32_t *kc32 = reinterpret_cast<const uint32_t *>(a.kc);
    // K as well: every load of the position goes out before the first wait
    uint32_t kw[NG];
    uint16_t ksr[NG];
    uint32_t kzr = 0;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        kw[g] = valid ? kc32[(slot * NG + g) * 4 + qd] : 0u;
        ksr[g] = valid ? a.ks[slot * NG + g] : (uint16_t)0;
        vw[g] = valid ? vc32[(slot * NG + g) * 4 + qd] : 0u;
        vsr[g] = (valid && qd == 0) ? a.vs[slot * NG + g] : (uint16_t)0;
    }
    if (valid) kzr = a.kz[slot];
    if (valid && qd == 0) vzr = a.vz[slot];
    // query rows of the group, FP32: every load issued before the first store
    constexpr int kQPer = (kMaxGroup * D + kAttnThreads - 1) / kAttnThreads;
    uint32_t qraw[kQPer];
    const uint16_t *qh = a.q + (size_t)h * grp * D;  // the group's rows are contiguous
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
        const int i = tid + u * kAttnThreads;
        qraw[u] = i < grp * D ? (uint32_t)qh[i] : 0u;
    }
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
        const int i = tid + u * kAttnThreads;
        if (i < grp * D) qs[i / D][i % D] = __uint_as_float(qraw[u] << 16);
    }
    __syncthreads();

    // 1. scores: word qd of every group, then the four partial sums of a position
    float s[GRP];
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi) s[gi] = 0.f;
    if (valid) {
        const uint32_t zw = kzr;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint32_t word = kw[g];
            const float sg = __half2float(__ushort_as_half(ksr[g]));
            const float nzs = -(float)((zw >> (4 * g)) & 0xFu) * sg;  // -z * s, exact
#pragma unroll
            for (int j4 = 0; j4 < 2; ++j4) {
                // channels 32g + 8qd + 4*j4 .. +3: (c - z) * s = fma(c, s, -z * s),
                // exact; c as a float by the 2^23 mantissa trick
                float kv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t code = (word >> (4 * (4 * j4 + u))) & 0xFu;
                    kv[u] = fmaf(__uint_as_float(0x4B000000u | code) - 8388608.f, sg, nzs);
                }
                const int d4 = (32 * g + 8 * qd + 4 * j4) / 4;
#pragma unroll
                for (int gi = 0; gi < GRP; ++gi)
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
    for (int gi = 0; gi < GRP; ++gi) {
        if (gi < grp) {
            // (q0 + q1) + (q2 + q3): the same order on all four threads
            s[gi] += __shfl_xor_sync(0xffffffffu, s[gi], 1);
            s[gi] += __shfl_xor_sync(0xffffffffu, s[gi], 2);
        }
    }
    if (qd == 0) {
#pragma unroll
        for (int gi = 0; gi < GRP; ++gi)
            if (gi < grp) sc[gi][pos] = valid ? s[gi] * a.scale : -INFINITY;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        vrec_s[(pos * NG + g) * 4 + qd] = vw[g];
        if (qd == 0) vsc_s[pos * NG + g] = vsr[g];
    }
    if (qd == 0) vz_s[pos] = vzr;
    __syncthreads();

    // 2. chunk maximum and sum per query head: the first 4 warps, a position
    //    per thread (warp shuffles, then the warps in order)
    if (warp < kStatWarps) {
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi) {
            if (gi >= grp) break;
            float m = sc[gi][tid];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) wmax[warp][gi] = m;
        }
    }
    __syncthreads();
    if (tid < grp) {
        float m = wmax[0][tid];
        for (int w = 1; w < kStatWarps; ++w) m = fmaxf(m, wmax[w][tid]);
        cm[tid] = m;
    }
    __syncthreads();
    if (warp < kStatWarps) {
        const int t2 = c * kChunk + tid;
#pragma unroll
        for (int gi = 0; gi < kMaxGroup; ++gi) {
            if (gi >= grp) break;
            const float p = t2 < a.T ? expf(sc[gi][tid] - cm[gi]) : 0.f;
            sc[gi][tid] = p;
            float l = p;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0) wsum[warp][gi] = l;
        }
    }
    __syncthreads();
    if (tid < grp) {
        float l = 0.f;
        for (int w = 0; w < kStatWarps; ++w) l += wsum[w][tid];
        cl[tid] = l;
    }

    // 3. weighted sum of V: warp w, positions 8w .. 8w + 7; lane l, channels l + 32g
    float acc[GRP][NG];
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi)
#pragma unroll
        for (int g = 0; g < NG; ++g) acc[gi][g] = 0.f;
    const int w8 = lane >> 3, sh = 4 * (lane & 7);
    const int nvalid = min(8, a.T - (c * kChunk + 8 * warp));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i >= nvalid) break;
        const int tl = 8 * warp + i;
        const uint32_t zw = vz_s[tl];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint32_t word = vrec_s[(tl * NG + g) * 4 + w8];
            const float sg = __half2float(__ushort_as_half(vsc_s[tl * NG + g]));
            const int z = (int)((zw >> (4 * g)) & 0xFu);
            const float vval = (float)((int)((word >> sh) & 0xFu) - z) * sg;
#pragma unroll
            for (int gi = 0; gi < GRP; ++gi)
                if (gi < grp) acc[gi][g] = fmaf(sc[gi][tl], vval, acc[gi][g]);
        }
    }
    // lane l holds channel 32g + 8*(l/8) + l%8 = 32g + l; the V stage is dead
    __syncthreads();
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi)
        if (gi < grp)
#pragma unroll
            for (int g = 0; g < NG; ++g) red[((size_t)warp * grp + gi) * D + 32 * g + lane] = acc[gi][g];
    __syncthreads();
    for (int i = tid; i < grp * D; i += kAttnThreads) {
        const int gi = i / D, d = i - gi * D;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) v += red[((size_t)w * grp + gi) * D + d];
        const size_t qi = (size_t)(h * grp + gi) * a.nch + c;
        a.ws_acc[qi * D + d] = v;
        if (d == 0) {
            a.ws_ml[2 * qi] = cm[gi];
            a.ws_ml[2 * qi + 1] = cl[gi];
        }
    }
}

// Merge of the chunk partials, one CTA per query head and slice of 32
// channels.  M (the largest chunk maximum) and L = sum_c exp(m_c - M) l_c
// come from fixed-order block reductions; warp w adds channel lane of the
// chunks c = w, w + 8, ... in order (coalesced 128-byte rows), and the eight
// warps' sums are added in warp order.
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;

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
    __shared__ float red[kMergeWarps];
    __shared__ float part[kMergeWarps][32];
    attn_pdl_wait();  // the chunk kernel's partials are complete
    const int i = blockIdx.x, d0 = 32 * blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nch = a.nch;
    const float *ml = a.ws_ml + (size_t)i * nch * 2;
    const float *acc = a.ws_acc + (size_t)i * nch * D + d0 + lane;
    // the first eight chunks of this warp (c = warp, warp + 8, ...) are loaded
    // together with the statistics, before the maximum is known
    float mv[8], av[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int c = warp + u * kMergeWarps;
        mv[u] = c < nch ? ml[2 * c] : -INFINITY;
        av[u] = c < nch ? acc[(size_t)c * D] : 0.f;
    }
    float m = -INFINITY, lraw[2] = {0.f, 0.f}, mraw[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int c = tid + u * kMergeThreads;
        if (c < nch) {
            mraw[u] = ml[2 * c];
            lraw[u] = ml[2 * c + 1];
        }
    }
    for (int c = tid; c < nch; c += kMergeThreads) m = fmaxf(m, ml[2 * c]);
    const float M = block_max(m, red);
    float l = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u)
        if (tid + u * kMergeThreads < nch) l += expf(mraw[u] - M) * lraw[u];
    for (int c = tid + 2 * kMergeThreads; c < nch; c += kMergeThreads) l += expf(ml[2 * c] - M) * ml[2 * c + 1];
    const float L = block_sum(l, red);
    float o = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
        if (warp + u * kMergeWarps < nch) o = fmaf(expf(mv[u] - M), av[u], o);
    // further chunks, eight loads in flight at a time
    for (int c0 = warp + 8 * kMergeWarps; c0 < nch; c0 += 8 * kMergeWarps) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = c0 + u * kMergeWarps;
            mv[u] = c < nch ? ml[2 * c] : -INFINITY;
            av[u] = c < nch ? acc[(size_t)c * D] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (c0 + u * kMergeWarps < nch) o = fmaf(expf(mv[u] - M), av[u], o);
    }
    part[warp][lane] = o;
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) t += part[w][lane];
        a.out[(size_t)i * D + d0 + lane] = t / L;
    }
}

template <int NG, int GRP>
cudaError_t launch_attn(const AttnArgs &args, cudaStream_t s) {
    const size_t smem = attn_smem_bytes(NG, args.grp);
    cudaError_t e = cudaFuncSetAttribute(attn_partial_kernel<NG, GRP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.nch, (unsigned)args.Hkv, 1);
    cfg.blockDim = dim3(kAttnThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_partial_kernel<NG, GRP>, args);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)args.Hq, (unsigned)NG, 1);
    cfg.blockDim = dim3(kMergeThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, attn_combine_kernel, args, 32 * NG);
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
    const int bucket = a.grp <= 2 ? 2 : (a.grp <= 4 ? 4 : 8);
    cudaError_t e;
    switch (k.head_dim / 32 * 16 + bucket) {
#define SPECTRA_ATTN_CASE(NG)                                      \
    case NG * 16 + 2: e = launch_attn<NG, 2>(a, s); break;         \
    case NG * 16 + 4: e = launch_attn<NG, 4>(a, s); break;         \
    case NG * 16 + 8: e = launch_attn<NG, 8>(a, s); break;
        SPECTRA_ATTN_CASE(1)
        SPECTRA_ATTN_CASE(2)
        SPECTRA_ATTN_CASE(3)
        SPECTRA_ATTN_CASE(4)
        SPECTRA_ATTN_CASE(5)
        SPECTRA_ATTN_CASE(6)
        SPECTRA_ATTN_CASE(7)
        SPECTRA_ATTN_CASE(8)
#undef SPECTRA_ATTN_CASE
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
