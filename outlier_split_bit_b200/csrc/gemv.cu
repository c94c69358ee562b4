// gemv.cu -- fused dequantise + matvec over RT32-packed weights (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph and highlight 4: the
// 4-bit Group-32 weights are decoded in registers inside the decode kernel,
// and the BF16 outlier channels are multiplied in the same pass.
//
// Work decomposition.  Lane r of a warp owns row r of a 32-row tile, so every
// x value a lane needs is a shared-memory broadcast and one warp-wide 16-byte
// load per group streams one contiguous 512-byte segment of codes.  The
// super-groups (8 groups = 256 columns) of a tile are split over P slices:
// `ppc` warps of a CTA times `cl` CTAs of a thread-block cluster; slice sums
// are reduced in a fixed order through shared memory and, across the
// cluster, distributed shared memory.  No workspace, no atomics.
//
// Inner loop per group (32 codes, one 16-byte record per lane):
//   A = (word & 0x0F0F0F0F) | 0x80808080, B = ((word >> 4) & ...) | ...;
//   one byte permute per code builds the FP32 value f = 1 + c/128
//   (exponent 127, code in mantissa bits 16..19); packed FP32x2 FMAs
//   accumulate sum_k f_k x_k.  With X_g = sum_k x_k,
//   sum_k (c_k - z) x_k = 128 * sum_k f_k x_k - (128 + z) * X_g,
//   so the zero point and the scale are applied once per group:
//   y += s * (128 * A_g - (128 + z) * X_g).
//
// Programmatic dependent launch: the kernel lets the next kernel on the
// stream launch as soon as all of its CTAs run, issues the loads of its first
// super-group of (constant) weights, then waits for the previous grid before
// it reads x or writes y.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace spectra {
namespace {

// CTA size limit per batch width: more accumulators need more registers.
template <int MB>
struct MaxWarps {
    static constexpr int value = 8;
};
constexpr int kSgBytes = 8 * 512 + 512 + 128;  // codes + scales + zeros of a warp per super-group
constexpr int kOctBytes = 512;                 // outlier bytes of a warp per octet

struct GemvArgs {
    const uint4 *codes;
    const uint4 *scales;
    const uint32_t *zeros;
    const uint4 *outw;
    const int32_t *oidx;
    const uint16_t *x;
    void *y;
    int n, k, m, G, S, O8, n_o, T;
    int ppc, tpc, cl;
    int ytype;
    int smem_sg, smem_oc;  // capacity of the x stage (super-groups, octets)
};

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream32(const uint32_t *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// f = 1 + c/128 from byte b of a pre-masked register (byte = 0x80 | c).
template <int b>
__device__ __forceinline__ float code_f(uint32_t a) {
    return __uint_as_float(__byte_perm(a, 0x3F000000u, 0x7054u | (b << 8)));
}

__device__ __forceinline__ int slice_begin(int total, int s, int P) {
    return (int)(((int64_t)total * s) / P);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Shared-memory x stage.  Bulk x is stored per group in the lane-broadcast
// order: position 8w + 4*(j & 1) + (j >> 1) holds column 8w + j, and the
// MB batch rows of one position are contiguous.
template <int MB>
struct Stage {
    float *xs;    // [smem_sg*8][32][MB]
    float *xsum;  // [smem_sg*8][MB]
    float *xo;    // [smem_oc*8][MB]
    float *red;   // [NW][32][MB]
    float *part;  // [tpc][32][MB]
};

template <int MB>
__device__ __forceinline__ Stage<MB> carve(float *sm, const GemvArgs &a, int nw) {
    Stage<MB> st;
    st.xs = sm;
    st.xsum = st.xs + (size_t)a.smem_sg * 8 * 32 * MB;
    st.xo = st.xsum + (size_t)a.smem_sg * 8 * MB;
    st.red = st.xo + (size_t)a.smem_oc * 8 * MB;
    st.part = st.red + (size_t)nw * 32 * MB;
    return st;
}

template <int MB>
__device__ void stage_x(const GemvArgs &a, const Stage<MB> &st, int csg0, int csg1, int coc0,
                        int coc1) {
    const int ng = 8 * (csg1 - csg0);
    const int chunks = MB * ng * 4;  // 8 columns per chunk
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const int m = c / (ng * 4);
        const int kc = c - m * ng * 4;
        const int gl = kc >> 2, w = kc & 3;
        const int g = 8 * csg0 + gl;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (g < a.G && m < a.m)
            v = *reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.k + 32 * g + 8 * w);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        float *dst = st.xs + (size_t)gl * 32 * MB;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float f = (j & 1) ? bf16_hi(u[j >> 1]) : bf16_lo(u[j >> 1]);
            const int pos = 8 * w + 4 * (j & 1) + (j >> 1);
            dst[pos * MB + m] = f;
        }
    }
    const int no = 8 * (coc1 - coc0);
    for (int c = threadIdx.x; c < no * MB; c += blockDim.x) {
        const int jl = c / MB, m = c - (c / MB) * MB;
        const int j = 8 * coc0 + jl;
        float f = 0.f;
        if (j < a.n_o && m < a.m) f = bf16_lo(a.x[(size_t)m * a.k + a.oidx[j]]);
        st.xo[jl * MB + m] = f;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < ng * MB; c += blockDim.x) {
        const int gl = c / MB, m = c - (c / MB) * MB;
        const float *src = st.xs + (size_t)gl * 32 * MB + m;
        float s = 0.f;
#pragma unroll 8
        for (int p = 0; p < 32; ++p) s += src[p * MB];
        st.xsum[c] = s;
    }
}

struct SgRegs {
    uint4 q[8];
    uint4 sc;
    uint32_t zw;
};

__device__ __forceinline__ void load_sg(SgRegs &r, const GemvArgs &a, int t, int sg, int lane) {
    const uint4 *cp = a.codes + ((size_t)t * a.G + 8 * sg) * 32 + lane;
    const int ng = min(8, a.G - 8 * sg);
    if (ng == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) r.q[i] = ld_stream(cp + i * 32);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            r.q[i] = (i < ng) ? ld_stream(cp + i * 32) : make_uint4(0u, 0u, 0u, 0u);
    }
    r.sc = ld_stream(a.scales + ((size_t)t * a.S + sg) * 32 + lane);
    r.zw = ld_stream32(a.zeros + ((size_t)t * a.S + sg) * 32 + lane);
}

// sum_k f_k x_k for one group, MB == 1.
__device__ __forceinline__ float group_dot1(const uint4 &q, const float *xg) {
    const float4 *x4 = reinterpret_cast<const float4 *>(xg);
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t A = (wv[w] & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t B = ((wv[w] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
        const float4 xa = x4[2 * w], xb = x4[2 * w + 1];
        a0 = __ffma2_rn(make_float2(code_f<0>(A), code_f<1>(A)), make_float2(xa.x, xa.y), a0);
        a1 = __ffma2_rn(make_float2(code_f<2>(A), code_f<3>(A)), make_float2(xa.z, xa.w), a1);
        a2 = __ffma2_rn(make_float2(code_f<0>(B), code_f<1>(B)), make_float2(xb.x, xb.y), a2);
        a3 = __ffma2_rn(make_float2(code_f<2>(B), code_f<3>(B)), make_float2(xb.z, xb.w), a3);
    }
    const float2 s = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
    return s.x + s.y;
}

// sum_k f_k x[m][k] for one group, MB > 1 (MB even): acc[m] for all rows.
template <int MB>
__device__ __forceinline__ void group_dotm(const uint4 &q, const float *xg, float *out) {
    float2 ea[MB / 2], eb[MB / 2];
#pragma unroll
    for (int i = 0; i < MB / 2; ++i) ea[i] = eb[i] = make_float2(0.f, 0.f);
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t A = (wv[w] & 0x0F0F0F0Fu) | 0x80808080u;
        const uint32_t B = ((wv[w] >> 4) & 0x0F0F0F0Fu) | 0x80808080u;
        float fa[4] = {code_f<0>(A), code_f<1>(A), code_f<2>(A), code_f<3>(A)};
        float fb[4] = {code_f<0>(B), code_f<1>(B), code_f<2>(B), code_f<3>(B)};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float2 *xa = reinterpret_cast<const float2 *>(xg + (8 * w + b) * MB);
            const float2 *xb = reinterpret_cast<const float2 *>(xg + (8 * w + 4 + b) * MB);
            const float2 fa2 = make_float2(fa[b], fa[b]);
            const float2 fb2 = make_float2(fb[b], fb[b]);
#pragma unroll
            for (int i = 0; i < MB / 2; ++i) {
                ea[i] = __ffma2_rn(fa2, xa[i], ea[i]);
                eb[i] = __ffma2_rn(fb2, xb[i], eb[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < MB / 2; ++i) {
        const float2 s = __fadd2_rn(ea[i], eb[i]);
        out[2 * i] = s.x;
        out[2 * i + 1] = s.y;
    }
}

template <int MB>
__device__ __forceinline__ void compute_sg(const SgRegs &r, const float *xs_sg,
                                           const float *xsum_sg, float *yacc) {
    const uint32_t scw[4] = {r.sc.x, r.sc.y, r.sc.z, r.sc.w};
#pragma unroll
    for (int gg = 0; gg < 8; ++gg) {
        const float s = __half2float(__ushort_as_half(
            (unsigned short)((gg & 1) ? (scw[gg >> 1] >> 16) : (scw[gg >> 1] & 0xFFFFu))));
        // 128 + z as a float: exponent of 128, z in mantissa bits 16..19
        const uint32_t zsh = (gg <= 4) ? (r.zw << (16 - 4 * gg)) : (r.zw >> (4 * gg - 16));
        const float zf = __uint_as_float((zsh & 0x000F0000u) | 0x43000000u);
        const float *xg = xs_sg + gg * 32 * MB;
        if constexpr (MB == 1) {
            const float Ag = group_dot1(r.q[gg], xg);
            const float tg = fmaf(128.f, Ag, -zf * xsum_sg[gg]);
            yacc[0] = fmaf(s, tg, yacc[0]);
        } else {
            float Ag[MB];
            group_dotm<MB>(r.q[gg], xg, Ag);
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                const float tg = fmaf(128.f, Ag[m], -zf * xsum_sg[gg * MB + m]);
                yacc[m] = fmaf(s, tg, yacc[m]);
            }
        }
    }
}

template <int MB>
__global__ void __launch_bounds__(MaxWarps<MB>::value * 32, 1) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) float smem[];
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cr = (a.cl > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int cid = blockIdx.x / a.cl;
    const int P = a.ppc * a.cl;
    const int tl = warp / a.ppc, sl = warp - (warp / a.ppc) * a.ppc;
    const int t = cid * a.tpc + tl;
    const bool active = t < a.T;
    const int slice = cr * a.ppc + sl;
    const int sg0 = slice_begin(a.S, slice, P), sg1 = slice_begin(a.S, slice + 1, P);
    const int oc0 = slice_begin(a.O8, slice, P), oc1 = slice_begin(a.O8, slice + 1, P);
    const int csg0 = slice_begin(a.S, cr * a.ppc, P), csg1 = slice_begin(a.S, (cr + 1) * a.ppc, P);
    const int coc0 = slice_begin(a.O8, cr * a.ppc, P),
              coc1 = slice_begin(a.O8, (cr + 1) * a.ppc, P);
    const Stage<MB> st = carve<MB>(smem, a, nw);

    pdl_launch_dependents();
    SgRegs ra, rb;
    if (active && sg0 < sg1) load_sg(ra, a, t, sg0, lane);
    pdl_wait();
    stage_x<MB>(a, st, csg0, csg1, coc0, coc1);
    __syncthreads();

    float yacc[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) yacc[m] = 0.f;
    if (active) {
        for (int sg = sg0; sg < sg1; sg += 2) {
            if (sg + 1 < sg1) load_sg(rb, a, t, sg + 1, lane);
            const int la = sg - csg0;
            compute_sg<MB>(ra, st.xs + (size_t)la * 8 * 32 * MB, st.xsum + la * 8 * MB, yacc);
            if (sg + 1 >= sg1) break;
            if (sg + 2 < sg1) load_sg(ra, a, t, sg + 2, lane);
            compute_sg<MB>(rb, st.xs + (size_t)(la + 1) * 8 * 32 * MB,
                           st.xsum + (la + 1) * 8 * MB, yacc);
        }
        for (int oc = oc0; oc < oc1; ++oc) {
            const uint4 ow = ld_stream(a.outw + ((size_t)t * a.O8 + oc) * 32 + lane);
            const uint32_t ov[4] = {ow.x, ow.y, ow.z, ow.w};
            const float *xo = st.xo + (size_t)(oc - coc0) * 8 * MB;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float wv = (e & 1) ? bf16_hi(ov[e >> 1]) : bf16_lo(ov[e >> 1]);
#pragma unroll
                for (int m = 0; m < MB; ++m) yacc[m] = fmaf(wv, xo[e * MB + m], yacc[m]);
            }
        }
    }

    // fixed-order reduction: slices of the CTA, then CTAs of the cluster
#pragma unroll
    for (int m = 0; m < MB; ++m) st.red[((size_t)warp * 32 + lane) * MB + m] = yacc[m];
    __syncthreads();
    float tot[MB];
    const bool leader = active && sl == 0;
    if (leader) {
#pragma unroll
        for (int m = 0; m < MB; ++m) tot[m] = 0.f;
        for (int s = 0; s < a.ppc; ++s) {
            const float *src = st.red + ((size_t)(tl * a.ppc + s) * 32 + lane) * MB;
#pragma unroll
            for (int m = 0; m < MB; ++m) tot[m] += src[m];
        }
    }
    if (a.cl > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        if (leader) {
#pragma unroll
            for (int m = 0; m < MB; ++m) st.part[((size_t)tl * 32 + lane) * MB + m] = tot[m];
        }
        cluster.sync();
        if (leader && cr == 0) {
#pragma unroll
            for (int m = 0; m < MB; ++m) tot[m] = 0.f;
            for (int rk = 0; rk < a.cl; ++rk) {
                const float *rp = cluster.map_shared_rank(st.part, rk) + ((size_t)tl * 32 + lane) * MB;
#pragma unroll
                for (int m = 0; m < MB; ++m) tot[m] += rp[m];
            }
        }
        cluster.sync();
    }
    if (leader && cr == 0) {
        const int row = 32 * t + lane;
        if (row < a.n) {
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                if (m < a.m) {
                    if (a.ytype == SPECTRA_F32)
                        reinterpret_cast<float *>(a.y)[(size_t)m * a.n + row] = tot[m];
                    else
                        reinterpret_cast<__nv_bfloat16 *>(a.y)[(size_t)m * a.n + row] =
                            __float2bfloat16_rn(tot[m]);
                }
            }
        }
    }
}

struct Plan {
    int ppc, tpc, cl, nw;
    int smem_sg, smem_oc;
    size_t smem;
    unsigned grid;
};

size_t smem_bytes(int MB, int smem_sg, int smem_oc, int nw, int tpc) {
    return sizeof(float) * ((size_t)smem_sg * 8 * 32 * MB + (size_t)smem_sg * 8 * MB +
                            (size_t)smem_oc * 8 * MB + (size_t)nw * 32 * MB + (size_t)tpc * 32 * MB);
}

int max_share(int total, int parts_per, int cl, int P) {
    // the largest CTA share of `total` units when P slices are grouped by `parts_per`
    int mx = 0;
    for (int c = 0; c < cl; ++c) {
        const int b = (int)(((int64_t)total * c * parts_per) / P);
        const int e = (int)(((int64_t)total * (c + 1) * parts_per) / P);
        if (e - b > mx) mx = e - b;
    }
    return mx;
}

// Pick slices per tile (P = ppc * cl) and tiles per CTA from a simple model:
// time ~ waves(T*P warps) * bytes of the largest slice, plus a small cost per
// reduction level.  Shared memory must hold the CTA's slice of x.
bool make_plan(const Geometry &g, int MB, int max_warps, const DeviceInfo &dev, Plan *out) {
    const int64_t warp_cap = (int64_t)dev.sm_count * 24;
    double best = 1e300;
    bool found = false;
    for (int cl = 1; cl <= 8; ++cl) {
        for (int ppc = 1; ppc <= max_warps; ++ppc) {
            const int P = ppc * cl;
            if (P > 1 && P > g.S) continue;
            const int tpc = (ppc >= 8) ? 1 : (g.T >= 2 * warp_cap / ppc ? 8 / ppc : 1);
            const int nw = tpc * ppc;
            if (nw > max_warps) continue;
            const int64_t warps = (int64_t)g.T * P;
            const int64_t waves = (warps + warp_cap - 1) / warp_cap;
            const int64_t slice_bytes = cdiv(g.S, P) * kSgBytes + cdiv(g.O8, P) * kOctBytes;
            const double cost = (double)waves * (double)slice_bytes + (ppc > 1 ? 1024.0 : 0.0) +
                                (cl > 1 ? 4096.0 + 512.0 * cl : 0.0);
            const int ssg = max_share(g.S, ppc, cl, P);
            const int soc = max_share(g.O8, ppc, cl, P);
            const size_t smem = smem_bytes(MB, ssg, soc, nw, tpc);
            if (smem > dev.smem_optin) continue;
            if (cost < best) {
                best = cost;
                found = true;
                out->ppc = ppc;
                out->tpc = tpc;
                out->cl = cl;
                out->nw = nw;
                out->smem_sg = ssg;
                out->smem_oc = soc;
                out->smem = smem;
                out->grid = (unsigned)(cdiv(g.T, tpc) * cl);
            }
        }
    }
    return found;
}

// Raise the dynamic shared-memory limit of one kernel instance, once per device.
template <int MB>
cudaError_t prepare_kernel(const DeviceInfo &dev) {
    static std::mutex mu;
    static bool done[64];
    std::lock_guard<std::mutex> lock(mu);
    if (dev.device >= 0 && dev.device < 64 && done[dev.device]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dev.smem_optin);
    if (e == cudaSuccess && dev.device >= 0 && dev.device < 64) done[dev.device] = true;
    return e;
}

template <int MB>
cudaError_t launch_mb(const GemvArgs &a, const Plan &p, const DeviceInfo &dev, cudaStream_t s) {
    cudaError_t pe = prepare_kernel<MB>(dev);
    if (pe != cudaSuccess) return pe;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(p.nw * 32, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (p.cl > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = p.cl;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<MB>, a);
}

}  // namespace

spectra_status launch_gemv(const spectra_layer &l, const uint16_t *x, int m, void *y, int ytype,
                           cudaStream_t s, const DeviceInfo &dev) {
    const Geometry g = Geometry::of(l.n, l.k, l.n_outliers);
    int done = 0;
    while (done < m) {
        const int mc = (m - done) > 8 ? 8 : (m - done);
        const int MB = mc == 1 ? 1 : (mc == 2 ? 2 : (mc <= 4 ? 4 : 8));
        Plan p;
        const int max_warps = MB <= 2 ? MaxWarps<1>::value : MaxWarps<8>::value;
        if (!make_plan(g, MB, max_warps, dev, &p)) return SPECTRA_ERR_SHAPE;
        GemvArgs a;
        a.codes = reinterpret_cast<const uint4 *>(l.codes);
        a.scales = reinterpret_cast<const uint4 *>(l.scales);
        a.zeros = l.zeros;
        a.outw = reinterpret_cast<const uint4 *>(l.outlier_w);
        a.oidx = l.outlier_idx;
        a.x = x + (size_t)done * l.k;
        a.y = (ytype == SPECTRA_F32)
                  ? (void *)(reinterpret_cast<float *>(y) + (size_t)done * l.n)
                  : (void *)(reinterpret_cast<uint16_t *>(y) + (size_t)done * l.n);
        a.n = l.n; a.k = l.k; a.m = mc;
        a.G = g.G; a.S = g.S; a.O8 = g.O8; a.n_o = g.n_o; a.T = g.T;
        a.ppc = p.ppc; a.tpc = p.tpc; a.cl = p.cl;
        a.ytype = ytype;
        a.smem_sg = p.smem_sg; a.smem_oc = p.smem_oc;
        cudaError_t e;
        switch (MB) {
            case 1: e = launch_mb<1>(a, p, dev, s); break;
            case 2: e = launch_mb<2>(a, p, dev, s); break;
            case 4: e = launch_mb<4>(a, p, dev, s); break;
            default: e = launch_mb<8>(a, p, dev, s); break;
        }
        if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
        done += mc;
    }
    return SPECTRA_OK;
}

}  // namespace spectra
