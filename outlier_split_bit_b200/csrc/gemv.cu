// gemv.cu -- fused dequantise + matvec over RT32-packed weights (sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph and highlight 4: the
// 4-bit Group-32 weights are decoded in registers inside the decode kernel,
// and the BF16 outlier channels are multiplied in the same pass.
//
// Work decomposition.  Lane r of a warp owns row r of a 32-row tile, so every
// x value a lane needs is a shared-memory broadcast, and one 16-byte record
// per lane per group makes the codes of a warp one contiguous 512-byte
// segment.  The work of a tile is a list of U units: its S super-groups (8
// groups = 256 columns: 4096 bytes of codes, 512 of scales, 128 of zero
// points) followed by its outlier batches (up to 8 octets of outlier columns,
// 4096 bytes).  The units of a tile are split evenly over P slices, each
// slice run by one warp; slice sums are reduced in a fixed order (shared
// memory, and distributed shared memory across a cluster), so results are
// bit-identical from run to run, with no workspace and no atomics.
//
// Inner loop per group (32 codes, one 16-byte record per lane): for each
// 32-bit word (8 codes, code j in nibble j) and s = 0..3, ONE logic op
//   p_s = ((word >> 4s) & 0x000F000F) | 0x43004300
// yields the BF16 pair (128 + c_s, 128 + c_{s+4}) -- BF16 has 7 mantissa
// bits, so 128 + c (c < 16) is exact -- and the mixed-precision FMA
// (fma.rn.f32.bf16: BF16 x BF16 products, FP32 accumulation) multiplies the
// pair by the matching BF16 pair of x straight from shared memory.  With
// X_g = sum_k x_k (FP32),
//   sum_k (c_k - z) x_k = sum_k (128 + c_k) x_k - (128 + z) X_g,
// so the zero point and the scale are applied once per group:
//   y += s * (A_g - (128 + z) X_g),  A_g = sum_k (128 + c_k) x_k.
// This keeps the integer pipe (half rate on sm_100) at ~0.9 operations per
// weight and puts the multiply-adds on the FMA pipe.
//
// Weight streaming: every warp owns a ring of D shared-memory stages, one
// unit per stage, filled by cp.async.bulk copies that complete on the
// stage's mbarrier.  Lane 0 keeps D units in flight; the warp waits on a
// stage (a bounded wait), decodes it from shared memory and refills it with
// the unit D ahead.
//
// Two launch shapes share this machinery:
//  - cluster kernel (one matrix, few tiles): a CTA runs `tpc` tiles x `ppc`
//    slices, a cluster of `cl` CTAs splits the units of the same tiles, and
//    rank 0 reduces the cluster through distributed shared memory;
//  - persistent kernel (one large matrix, or many independent matrices): one
//    16-warp CTA per SM, each walking a byte-balanced contiguous range of
//    work items (tpc tiles x ppc slices of one matrix); the rings keep
//    prefetching across item boundaries and x is restaged only when the
//    matrix changes.
// Programmatic dependent launch: a kernel lets the next kernel on the stream
// launch once all of its CTAs run, issues its first units of (constant)
// weights, and only then waits for the previous grid before it reads x or
// writes y; x's first loads go out before the rest of the ring is filled.
#include "stream.cuh"

namespace spectra {
namespace {

constexpr int kClusterWarps = 8;               // warps per CTA of the cluster kernel
constexpr int kPersistWarps = 16;              // warps per CTA of the persistent kernel
constexpr int kMaxCtas = 320;                  // persistent grid bound (2 x SMs of a B200 + margin)
constexpr size_t kChainWorkspace = 16;         // the chain kernel's completion counter (+ padding)

// Launch-wide shared-memory geometry.
struct Smem {
    int depth;  // ring stages per warp
    int xg;     // x-stage capacity in groups
    int xo;     // x-stage capacity in outlier slots
    int tpc;    // partial-sum rows (tiles) for the cluster reduction
};

struct ClusterArgs {
    Prob p;
    Smem sm;
    int pre;  // ring stages a warp issues before waiting on the previous grid
};

// Parameters of the persistent kernel, passed by value (kernel parameter space).
struct PersistArgs {
    Smem sm;
    int pre;                        // ring stages a warp issues before the wait
    int count;                      // problems
    int item_start[kMaxBatch + 1];  // first item of each problem
    int cta_first[kMaxCtas + 1];    // first item of each CTA
    Prob probs[kMaxBatch];
};
static_assert(sizeof(PersistArgs) <= 32760, "kernel parameter space");

// ---------------------------------------------------------------- shared memory

// Shared-memory layout of one CTA.  Bulk x is stored per group as 16 BF16
// pairs in the order the decoder pairs the codes: pair 4w + s holds
// (x_{8w+s}, x_{8w+s+4}); the MB batch rows of one pair are contiguous.
template <int MB>
struct Stage {
    uint8_t *ring;  // [nw][depth][kStageBytes]
    uint64_t *bar;  // [nw][depth]
    uint32_t *xs;   // [xg][16 pairs][MB]: BF16 pairs (x_{8w+s}, x_{8w+s+4}), pair 4w+s
    float *xsum;    // [xg][MB]
    uint32_t *xo;   // [xo/2][MB]: BF16 pairs of outlier slots (2i, 2i+1)
    float *red;     // [2][nw][32][MB]
    float *part;    // [tpc][32][MB]
};

__host__ __device__ inline size_t ring_bytes(int nw, int depth) {
    return (size_t)nw * depth * kStageBytes + (size_t)((nw * depth + 1) & ~1) * 8;
}

__host__ __device__ inline size_t stage_bytes(int MB, int nw, const Smem &s) {
    return ring_bytes(nw, s.depth) +
           sizeof(float) * ((size_t)s.xg * 16 * MB + (size_t)s.xg * MB + (size_t)s.xo / 2 * MB +
                            (size_t)2 * nw * 32 * MB + (size_t)s.tpc * 32 * MB);
}

template <int MB>
__device__ __forceinline__ Stage<MB> carve(float *sm, const Smem &s, int nw) {
    Stage<MB> st;
    st.ring = reinterpret_cast<uint8_t *>(sm);
    st.bar = reinterpret_cast<uint64_t *>(st.ring + (size_t)nw * s.depth * kStageBytes);
    st.xs = reinterpret_cast<uint32_t *>(st.bar + ((nw * s.depth + 1) & ~1));
    st.xsum = reinterpret_cast<float *>(st.xs + (size_t)s.xg * 16 * MB);
    st.xo = reinterpret_cast<uint32_t *>(st.xsum + (size_t)s.xg * MB);
    st.red = reinterpret_cast<float *>(st.xo + (size_t)s.xo / 2 * MB);
    st.part = st.red + (size_t)2 * nw * 32 * MB;
    return st;
}

// A slice of a tile: its super-groups and its outlier batches, each split
// evenly over the P slices so that every slice has the same mix of work.
struct Slice {
    int sg0, nsg;  // super-groups [sg0, sg0 + nsg)
    int ob0, nob;  // outlier batches [ob0, ob0 + nob)
};

__device__ __forceinline__ Slice slice_of(const Prob &a, int s, int P) {
    const int OB = a.U - a.S;
    Slice r;
    r.sg0 = split_at(a.S, s, P);
    r.nsg = split_at(a.S, s + 1, P) - r.sg0;
    r.ob0 = split_at(OB, s, P);
    r.nob = split_at(OB, s + 1, P) - r.ob0;
    return r;
}

// slice_of for P = 2^lg slices (shifts instead of divisions).
__device__ __forceinline__ Slice slice_of_pow2(const Prob &a, int s, int lg) {
    const int OB = a.U - a.S;
    Slice r;
    r.sg0 = (a.S * s) >> lg;
    r.nsg = ((a.S * (s + 1)) >> lg) - r.sg0;
    r.ob0 = (OB * s) >> lg;
    r.nob = ((OB * (s + 1)) >> lg) - r.ob0;
    return r;
}

// Local unit u of a slice -> unit id (super-group id, or S + batch id).
__device__ __forceinline__ int unit_id(const Prob &a, const Slice &sl, int u) {
    return u < sl.nsg ? sl.sg0 + u : a.S + sl.ob0 + (u - sl.nsg);
}

// x staged for slices [s0, s1) of P: groups and outlier slots.
struct XRange {
    int g0, g1;  // groups [g0, g1) (g1 may pass G: padding groups)
    int j0, j1;  // outlier slots [j0, j1) (j1 may pass n_o: padding slots)
};

__device__ __forceinline__ XRange x_range(const Prob &a, int s0, int s1, int P) {
    const int OB = a.U - a.S;
    XRange r;
    r.g0 = 8 * split_at(a.S, s0, P);
    r.g1 = 8 * split_at(a.S, s1, P);
    r.j0 = 8 * kOB * split_at(OB, s0, P);
    r.j1 = 8 * kOB * split_at(OB, s1, P);
    return r;
}

// Column indices of the first round of outlier slots a thread gathers (8
// pairs per thread in flight).  They are part of the packed layer, not an
// output of the previous kernel, so they may be loaded before the wait on it.
struct XIdx {
    int i0[8], i1[8];
};

__device__ __forceinline__ void load_x_idx(const Prob &a, const XRange &xr, int MB, XIdx &xi) {
    const int np = (xr.j1 - xr.j0) / 2;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + i * blockDim.x;
        const int j = xr.j0 + 2 * (c / MB);
        const bool ok = c < np * MB;
        xi.i0[i] = (ok && j < a.n_o) ? a.oidx[j] : -1;
        xi.i1[i] = (ok && j + 1 < a.n_o) ? a.oidx[j + 1] : -1;
    }
}

// The first round of a thread's x loads, held in registers: the first bulk
// round (4 x 16 bytes of one group) and the first gather round (8 outlier
// pairs).  Loading them before the kernel issues its remaining weight stages
// puts them ahead of those stages in the memory system's queues.
struct XFirst {
    uint4 v0[4];
    uint32_t lo[8], hi[8];
};

template <int MB, bool kL2>
__device__ __forceinline__ void stage_x_load(const Prob &a, const XRange &xr, const XIdx &xi,
                                             XFirst &f) {
    const int nth = blockDim.x;
    const int ng = xr.g1 - xr.g0;
    const int np = (xr.j1 - xr.j0) / 2;
    {
        const int c = threadIdx.x, gl = c / MB, m = c - gl * MB, g = xr.g0 + gl;
        if (c < ng * MB && g < a.G && m < a.m) {
            if (a.bidx == nullptr) {
                const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.kx + 32 * g);
#pragma unroll
                for (int w = 0; w < 4; ++w) f.v0[w] = ld_x<kL2>(src + w);
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) f.v0[w] = bulk_x8_gather<kL2>(a, m, 32 * g + 8 * w);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + i * nth;
        const int m = c % MB;
        const bool mv = c < np * MB && m < a.m;
        f.lo[i] = (mv && xi.i0[i] >= 0) ? ld_x<kL2>(a.x + (size_t)m * a.kx + xi.i0[i]) : 0u;
        f.hi[i] = (mv && xi.i1[i] >= 0) ? ld_x<kL2>(a.x + (size_t)m * a.kx + xi.i1[i]) : 0u;
    }
}

// Stage x for a unit range: bulk groups as BF16 pairs in the decoder's order
// with their FP32 sums X_g (column order), and the BF16 pairs of the outlier
// slots, gathered through the index list; the first round comes from `f`.
template <int MB, bool kL2>
__device__ void stage_x_store(const Prob &a, const Stage<MB> &st, const XRange &xr,
                              const XFirst &f) {
    const int nth = blockDim.x;
    const int ng = xr.g1 - xr.g0;
    const int np = (xr.j1 - xr.j0) / 2;
    for (int c = threadIdx.x; c < ng * MB; c += nth) {
        const int gl = c / MB, m = c - gl * MB;
        const int g = xr.g0 + gl;
        uint32_t *dst = st.xs + (size_t)gl * 16 * MB + m;
        float sum = 0.f;
        if (g < a.G && m < a.m) {
            uint4 v[4];
            if (c == (int)threadIdx.x) {
#pragma unroll
                for (int w = 0; w < 4; ++w) v[w] = f.v0[w];
            } else if (a.bidx == nullptr) {
                const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.kx + 32 * g);
#pragma unroll
                for (int w = 0; w < 4; ++w) v[w] = ld_x<kL2>(src + w);
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) v[w] = bulk_x8_gather<kL2>(a, m, 32 * g + 8 * w);
            }
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t u[4] = {v[w].x, v[w].y, v[w].z, v[w].w};
                // u[i] holds columns 8w + 2i (low half) and 8w + 2i + 1 (high half)
                uint32_t h[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) h[j] = (j & 1) ? (u[j >> 1] >> 16) : (u[j >> 1] & 0xFFFFu);
#pragma unroll
                for (int j = 0; j < 8; ++j) sum += __uint_as_float(h[j] << 16);
#pragma unroll
                for (int sp = 0; sp < 4; ++sp) dst[(4 * w + sp) * MB] = h[sp] | (h[sp + 4] << 16);
            }
        } else {
#pragma unroll
            for (int p = 0; p < 16; ++p) dst[p * MB] = 0u;
        }
        st.xsum[c] = sum;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + i * nth;
        if (c < np * MB) st.xo[c] = f.lo[i] | (f.hi[i] << 16);
    }
    // further gather rounds: 8 pairs per thread in flight
    for (int base = 8 * nth; base < np * MB; base += 8 * nth) {
        int i0[8], i1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = base + threadIdx.x + i * nth;
            const int j = xr.j0 + 2 * (c / MB);
            const bool ok = c < np * MB;
            i0[i] = (ok && j < a.n_o) ? a.oidx[j] : -1;
            i1[i] = (ok && j + 1 < a.n_o) ? a.oidx[j + 1] : -1;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = base + threadIdx.x + i * nth;
            if (c < np * MB) {
                const int m = c % MB;
                const bool mv = m < a.m;
                const uint32_t l = (i0[i] >= 0 && mv) ? ld_x<kL2>(a.x + (size_t)m * a.kx + i0[i]) : 0u;
                const uint32_t h = (i1[i] >= 0 && mv) ? ld_x<kL2>(a.x + (size_t)m * a.kx + i1[i]) : 0u;
                st.xo[c] = l | (h << 16);
            }
        }
    }
}

template <int MB, bool kL2>
__device__ __forceinline__ void stage_x(const Prob &a, const Stage<MB> &st, const XRange &xr,
                                        const XIdx &xi) {
    XFirst f;
    stage_x_load<MB, kL2>(a, xr, xi, f);
    stage_x_store<MB, kL2>(a, st, xr, f);
}

// ---------------------------------------------------------------- units

// lo += c.lo * x.lo, hi += c.hi * x.hi: BF16 products, FP32 accumulation.
__device__ __forceinline__ void mfma2(float &lo, float &hi, uint32_t c, uint32_t x) {
    asm("{\n\t.reg .b16 cl, ch, xl, xh;\n\t"
        "mov.b32 {cl, ch}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, cl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %1, ch, xh, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(c), "r"(x));
}

// A_g[m] = sum_k (128 + c_k) x[m][k] for one group.
template <int MB>
__device__ __forceinline__ void group_dot(const uint4 &q, const uint32_t *xg, float *out) {
    float acc[MB][4];
#pragma unroll
    for (int m = 0; m < MB; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t cp[4] = {code_pair<0>(wv[w]), code_pair<1>(wv[w]), code_pair<2>(wv[w]),
                                code_pair<3>(wv[w])};
        if constexpr (MB == 1) {
            const uint4 xw = *reinterpret_cast<const uint4 *>(xg + 4 * w);
            mfma2(acc[0][0], acc[0][1], cp[0], xw.x);
            mfma2(acc[0][2], acc[0][3], cp[1], xw.y);
            mfma2(acc[0][0], acc[0][1], cp[2], xw.z);
            mfma2(acc[0][2], acc[0][3], cp[3], xw.w);
        } else {
#pragma unroll
            for (int sp = 0; sp < 4; ++sp) {
                const uint32_t *xp = xg + (4 * w + sp) * MB;
#pragma unroll
                for (int m = 0; m < MB; m += 2) {
                    const uint2 x2 = *reinterpret_cast<const uint2 *>(xp + m);
                    mfma2(acc[m][sp & 1], acc[m][2 + (sp & 1)], cp[sp], x2.x);
                    mfma2(acc[m + 1][sp & 1], acc[m + 1][2 + (sp & 1)], cp[sp], x2.y);
                }
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) out[m] = (acc[m][0] + acc[m][1]) + (acc[m][2] + acc[m][3]);
}

template <int MB>
__device__ __forceinline__ void compute_group(const uint8_t *stage, int gg, int lane,
                                              const uint32_t *scw, uint32_t zw,
                                              const uint32_t *xs_sg, const float *xsum_sg,
                                              float *yacc) {
    const uint4 q = *reinterpret_cast<const uint4 *>(stage + gg * 512 + lane * 16);
    const float s = __half2float(__ushort_as_half(
        (unsigned short)((gg & 1) ? (scw[gg >> 1] >> 16) : (scw[gg >> 1] & 0xFFFFu))));
    // 128 + z as a float: exponent of 128, z in mantissa bits 16..19
    const uint32_t zsh = (gg <= 4) ? (zw << (16 - 4 * gg)) : (zw >> (4 * gg - 16));
    const float zf = __uint_as_float((zsh & 0x000F0000u) | 0x43000000u);
    float Ag[MB];
    group_dot<MB>(q, xs_sg + gg * 16 * MB, Ag);
#pragma unroll
    for (int m = 0; m < MB; ++m) yacc[m] = fmaf(s, fmaf(-zf, xsum_sg[gg * MB + m], Ag[m]), yacc[m]);
}

template <int MB>
__device__ __forceinline__ void compute_sg(const uint8_t *stage, int ng, int lane,
                                           const uint32_t *xs_sg, const float *xsum_in,
                                           float *yacc) {
    // the group sums of the super-group: for MB <= 2 vector loads into
    // registers, for wider batches straight from shared memory
    constexpr int kRegSums = MB <= 2 ? 8 * MB : 1;
    float xsum_reg[kRegSums];
    if constexpr (MB <= 2) {
#pragma unroll
        for (int i = 0; i < 2 * MB; ++i) {
            const float4 v = reinterpret_cast<const float4 *>(xsum_in)[i];
            xsum_reg[4 * i] = v.x;
            xsum_reg[4 * i + 1] = v.y;
            xsum_reg[4 * i + 2] = v.z;
            xsum_reg[4 * i + 3] = v.w;
        }
    }
    const float *xsum_sg = MB <= 2 ? xsum_reg : xsum_in;
    const uint4 sc = *reinterpret_cast<const uint4 *>(stage + 4096 + lane * 16);
    const uint32_t zw = *reinterpret_cast<const uint32_t *>(stage + 4608 + lane * 4);
    const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
    if (ng == 8) {
        // full super-group: straight-line code, the 8 groups overlap
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) compute_group<MB>(stage, gg, lane, scw, zw, xs_sg, xsum_sg, yacc);
    } else {
#pragma unroll
        for (int gg = 0; gg < 8; ++gg)
            if (gg < ng) compute_group<MB>(stage, gg, lane, scw, zw, xs_sg, xsum_sg, yacc);
    }
}

// Outlier octets: BF16 weight pairs times BF16 x pairs, FP32 accumulation.
template <int MB>
__device__ __forceinline__ void compute_ob(const uint8_t *stage, int lane, const uint32_t *xo,
                                           int n_valid, float *yacc) {
    float lo[MB], hi[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) lo[m] = hi[m] = 0.f;
#pragma unroll
    for (int i = 0; i < kOB; ++i) {
        if (i >= n_valid) break;
        const uint4 w4 = *reinterpret_cast<const uint4 *>(stage + i * 512 + lane * 16);
        const uint32_t wp[4] = {w4.x, w4.y, w4.z, w4.w};
        const uint32_t *xi = xo + i * 4 * MB;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int m = 0; m < MB; ++m) mfma2(lo[m], hi[m], wp[e], xi[e * MB + m]);
        }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) yacc[m] += lo[m] + hi[m];
}

// Decode unit u from a ring stage against the staged x of range xr.
template <int MB>
__device__ __forceinline__ void compute_unit(const Prob &a, const uint8_t *stage, int lane,
                                             const Stage<MB> &st, const XRange &xr, int u,
                                             float *yacc) {
    if (u < a.S) {
        const int l = 8 * u - xr.g0;  // local index of the super-group's first group
        compute_sg<MB>(stage, min(8, a.G - 8 * u), lane, st.xs + (size_t)l * 16 * MB,
                       st.xsum + l * MB, yacc);
    } else {
        const int b = u - a.S;
        compute_ob<MB>(stage, lane, st.xo + (size_t)((8 * kOB * b - xr.j0) / 2) * MB,
                       min(kOB, a.O8 - kOB * b), yacc);
    }
}

// ---------------------------------------------------------------- cluster kernel

// One matrix: CTA = tpc tiles x ppc slices, cluster of cl CTAs along the units.
template <int MB>
__global__ void __launch_bounds__(kClusterWarps * 32, MB == 1 ? 2 : 1)
    gemv_cluster_kernel(const ClusterArgs args) {
    extern __shared__ __align__(16) float smem[];
    const Prob &a = args.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cr = (a.cl > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int cid = blockIdx.x / a.cl;
    const int P = a.ppc * a.cl;
    const int tl = warp / a.ppc, sl = warp - tl * a.ppc;
    const int t = cid * a.tpc + tl;
    const bool active = tl < a.tpc && t < a.T;
    const Slice slc = slice_of(a, cr * a.ppc + sl, P);
    const int nunits = active ? slc.nsg + slc.nob : 0;
    const XRange xr = x_range(a, cr * a.ppc, (cr + 1) * a.ppc, P);
    const Stage<MB> st = carve<MB>(smem, args.sm, kClusterWarps);

    Ring ring;
    ring_init(ring, st.ring + (size_t)warp * args.sm.depth * kStageBytes,
              st.bar + warp * args.sm.depth, args.sm.depth, lane);
    pdl_launch_dependents();
    // `pre` stages cover the wait; the rest are issued behind x's first loads
    const int pre = min(args.pre, ring.D);
    int next = 0;
    for (; next < nunits && next < pre; ++next) ring_issue(ring, a, t, unit_id(a, slc, next), lane);
    XIdx xi;
    load_x_idx(a, xr, MB, xi);
    pdl_wait();
    XFirst xf;
    stage_x_load<MB, false>(a, xr, xi, xf);
    for (; next < nunits && next < ring.D; ++next) ring_issue(ring, a, t, unit_id(a, slc, next), lane);
    stage_x_store<MB, false>(a, st, xr, xf);
    __syncthreads();

    float yacc[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) yacc[m] = 0.f;
    for (int u = 0; u < nunits; ++u) {
        const uint8_t *stage = ring_acquire(ring, lane);
        if (stage) compute_unit<MB>(a, stage, lane, st, xr, unit_id(a, slc, u), yacc);
        ring_release(ring);
        if (next < nunits) ring_issue(ring, a, t, unit_id(a, slc, next++), lane);
    }
    ring_drain(ring);

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
                const float *rp =
                    cluster.map_shared_rank(st.part, rk) + ((size_t)tl * 32 + lane) * MB;
#pragma unroll
                for (int m = 0; m < MB; ++m) tot[m] += rp[m];
            }
        }
        cluster.sync();
    }
    if (leader && cr == 0) {
#pragma unroll
        for (int m = 0; m < MB; ++m) store_y(a, t, lane, m, tot[m]);
    }
}

// ---------------------------------------------------------------- persistent kernel

__device__ __forceinline__ int prob_of(const PersistArgs &args, int item) {
    int lo = 0, hi = args.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (args.item_start[mid] <= item)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Where one warp's issue pointer stands: item, its problem, tile, slice and
// local unit.
struct Cursor {
    int item, p, t, u;
    Slice sl;
};

// Problem of `item`, searched forward from `p` (items only increase).
__device__ __forceinline__ int prob_from(const PersistArgs &args, int item, int p) {
    while (p + 1 < args.count && args.item_start[p + 1] <= item) ++p;
    return p;
}

// Move the cursor to the first unit of `c.item` or of a later item of this warp.
__device__ __forceinline__ void cursor_load(const PersistArgs &args, int it1, int warp, Cursor &c) {
    while (c.item < it1) {
        c.p = prob_from(args, c.item, c.p);
        const Prob &a = args.probs[c.p];
        const int blk = c.item - args.item_start[c.p];
        const int tl = warp >> a.lgp;
        c.t = blk * a.tpc + tl;
        if (c.t < a.T) {
            c.sl = slice_of_pow2(a, warp & (a.ppc - 1), a.lgp);
            c.u = 0;
            if (c.sl.nsg + c.sl.nob > 0) return;
        }
        ++c.item;
    }
}

__device__ __forceinline__ void cursor_next(const PersistArgs &args, int it1, int warp, Cursor &c) {
    if (++c.u < c.sl.nsg + c.sl.nob) return;
    ++c.item;
    cursor_load(args, it1, warp, c);
}

__device__ __forceinline__ void cursor_issue(const PersistArgs &args, Ring &ring, const Cursor &c,
                                             int lane) {
    const Prob &a = args.probs[c.p];
    ring_issue(ring, a, c.t, unit_id(a, c.sl, c.u), lane);
}

template <int MB>
__global__ void __launch_bounds__(kPersistWarps * 32, 1)
    gemv_persistent_kernel(const PersistArgs args) {
    extern __shared__ __align__(16) float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int it0 = args.cta_first[blockIdx.x], it1 = args.cta_first[blockIdx.x + 1];
    const Stage<MB> st = carve<MB>(smem, args.sm, kPersistWarps);

    Ring ring;
    ring_init(ring, st.ring + (size_t)warp * args.sm.depth * kStageBytes,
              st.bar + warp * args.sm.depth, args.sm.depth, lane);
    pdl_launch_dependents();
    Cursor ic;
    ic.item = it0;
    ic.p = it0 < it1 ? prob_of(args, it0) : 0;
    cursor_load(args, it1, warp, ic);
    // `pre` stages cover the wait; the rest are issued behind x's first loads
    const int pre = min(args.pre, ring.D);
    int d = 0;
    for (; d < pre && ic.item < it1; ++d) {
        cursor_issue(args, ring, ic, lane);
        cursor_next(args, it1, warp, ic);
    }
    int p = it0 < it1 ? prob_of(args, it0) : 0;
    int cur_p = -1;
    XRange xr = {0, 0, 0, 0};
    XIdx xi;
    if (it0 < it1) {
        xr = x_range(args.probs[p], 0, 1, 1);
        load_x_idx(args.probs[p], xr, MB, xi);
    }
    pdl_wait();
    if (it0 < it1) {
        XFirst xf;
        stage_x_load<MB, false>(args.probs[p], xr, xi, xf);
        for (; d < ring.D && ic.item < it1; ++d) {
            cursor_issue(args, ring, ic, lane);
            cursor_next(args, it1, warp, ic);
        }
        stage_x_store<MB, false>(args.probs[p], st, xr, xf);
        __syncthreads();
        cur_p = p;
    }

    int rbuf = 0;
    for (int item = it0; item < it1; ++item) {
        p = prob_from(args, item, p);
        const Prob &a = args.probs[p];
        if (p != cur_p) {
            // every warp is done with the previous x (the branch is CTA-uniform)
            __syncthreads();
            xr = x_range(a, 0, 1, 1);
            XIdx xi;
            load_x_idx(a, xr, MB, xi);
            stage_x<MB, false>(a, st, xr, xi);
            __syncthreads();
            cur_p = p;
        }
        const int blk = item - args.item_start[p];
        const int tl = warp >> a.lgp, sl = warp & (a.ppc - 1);
        const int t = blk * a.tpc + tl;
        const bool active = t < a.T;
        const Slice slc = slice_of_pow2(a, sl, a.lgp);
        const int nunits = active ? slc.nsg + slc.nob : 0;
        float yacc[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) yacc[m] = 0.f;
        for (int u = 0; u < nunits; ++u) {
            const uint8_t *stage = ring_acquire(ring, lane);
            if (stage) compute_unit<MB>(a, stage, lane, st, xr, unit_id(a, slc, u), yacc);
            ring_release(ring);
            if (ic.item < it1) {
                cursor_issue(args, ring, ic, lane);
                cursor_next(args, it1, warp, ic);
            }
        }
        if (a.ppc == 1) {
            if (active) {
#pragma unroll
                for (int m = 0; m < MB; ++m) store_y(a, t, lane, m, yacc[m]);
            }
        } else {
            // the ppc warps of one tile meet on their own barrier (ids 1..tpc)
            float *red = st.red + (size_t)rbuf * kPersistWarps * 32 * MB;
#pragma unroll
            for (int m = 0; m < MB; ++m) red[((size_t)warp * 32 + lane) * MB + m] = yacc[m];
            named_sync(1 + tl, 32 * a.ppc);
            if (active && sl == 0) {
#pragma unroll
                for (int m = 0; m < MB; ++m) {
                    float tot = 0.f;
                    for (int s = 0; s < a.ppc; ++s)
                        tot += red[((size_t)(tl * a.ppc + s) * 32 + lane) * MB + m];
                    store_y(a, t, lane, m, tot);
                }
            }
            rbuf ^= 1;
        }
    }
    ring_drain(ring);
}

// ---------------------------------------------------------------- chain kernel
//
// A sequence of batch-1 matvecs where problem i may read what problems
// before it wrote (x of one layer = y of the last): one launch of one 16-warp
// CTA per SM, all resident at once.  Every problem is spread over all CTAs
// (CTA c takes its items c, c + ncta, ...), and before a CTA reads x of
// problem i it waits until every CTA has counted the problems before i's
// stage as done on a global counter (release / acquire at GPU scope); the
// problems of one stage (q, k and v of a layer share their input) run
// without a wait between them.  The weight rings keep
// prefetching across problems while a CTA waits, so the weight stream
// overlaps the wait.  An item is tpc tiles x ppc slices (tpc x ppc = 16
// warps); a tile's units are cut into contiguous slices, so the busiest warp
// of a small problem holds as few units as the problem allows (a lone warp
// decodes a unit in about a microsecond).

struct ChainArgs {
    Smem sm;
    int count;                // problems
    unsigned int *done;       // completion counter (zeroed before the launch)
    // problems that must be complete before problem p reads x: the index of
    // the first problem of p's stage (p itself when every problem is a stage)
    uint16_t need[kMaxBatch];
    // items of the earlier problems of p's stage: a stage's items are dealt
    // over the CTAs as one list, so its problems run on different CTAs
    int base[kMaxBatch];
    Prob probs[kMaxBatch];    // each with its own item shape (ppc x tpc = 16 warps)
};
static_assert(sizeof(ChainArgs) <= 32760, "kernel parameter space");

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait until *ctr >= target; bounded like the ring waits (one second of
// %globaltimer time), sleeping between polls.  Returns false on a timeout.
__device__ __forceinline__ bool counter_wait(const unsigned int *ctr, unsigned int target) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kWaitRounds; ++i) {
        __nanosleep(64);
        if (ld_acquire_gpu(ctr) >= target) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
    return false;
}

// Slice s of P of a tile as a contiguous range of its unit list
// (super-groups, then outlier batches): with P >= U every slice has at most
// one unit.
__device__ __forceinline__ Slice slice_contig(const Prob &a, int s, int P) {
    const int u0 = split_at(a.U, s, P), u1 = split_at(a.U, s + 1, P);
    Slice r;
    r.sg0 = u0;
    r.nsg = max(0, min(u1, a.S) - u0);
    r.ob0 = max(u0, a.S) - a.S;
    r.nob = u1 - u0 - r.nsg;
    return r;
}

// The tile and slice of warp `warp` in item `item` of a problem.
struct ChainWork {
    int t, tl, sl;
    Slice slc;
};

__device__ __forceinline__ ChainWork chain_work(const Prob &a, int item, int warp) {
    ChainWork w;
    w.tl = warp / a.ppc;
    w.sl = warp - w.tl * a.ppc;
    w.t = item * a.tpc + w.tl;
    w.slc = slice_contig(a, w.sl, a.ppc);
    return w;
}

// This CTA's first item of problem p (its later ones follow every gridDim.x):
// item i of p is item base[p] + i of its stage's list, dealt round robin.
__device__ __forceinline__ int chain_first(const ChainArgs &args, int p) {
    const int n = (int)gridDim.x;
    const int i0 = ((int)blockIdx.x - args.base[p]) % n;
    return i0 < 0 ? i0 + n : i0;
}

// One warp's position in the chain's unit sequence.
struct ChainCursor {
    int p, item, u;
    ChainWork w;
};

// Move the cursor to the first unit at or after (c.p, c.item) that this warp
// owns.
__device__ __forceinline__ void chain_load(const ChainArgs &args, int warp, ChainCursor &c) {
    while (c.p < args.count) {
        const Prob &a = args.probs[c.p];
        if (c.item < a.items) {
            c.w = chain_work(a, c.item, warp);
            c.u = 0;
            if (c.w.t < a.T && c.w.slc.nsg + c.w.slc.nob > 0) return;
            c.item += gridDim.x;
        } else {
            ++c.p;
            if (c.p < args.count) c.item = chain_first(args, c.p);
        }
    }
}

__device__ __forceinline__ void chain_next(const ChainArgs &args, int warp, ChainCursor &c) {
    if (++c.u < c.w.slc.nsg + c.w.slc.nob) return;
    c.item += gridDim.x;
    chain_load(args, warp, c);
}

__global__ void __launch_bounds__(kPersistWarps * 32, 1) gemv_chain_kernel(const ChainArgs args) {
    extern __shared__ __align__(16) float smem[];
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Stage<1> st = carve<1>(smem, args.sm, kPersistWarps);
    if (threadIdx.x == 1) s_abort = 0;
    Ring ring;
    ring_init(ring, st.ring + (size_t)warp * args.sm.depth * kStageBytes,
              st.bar + warp * args.sm.depth, args.sm.depth, lane);
    // weights are constant: the ring is filled before any wait
    ChainCursor ic;
    ic.p = 0;
    ic.item = chain_first(args, 0);
    chain_load(args, warp, ic);
    for (int d = 0; d < ring.D && ic.p < args.count; ++d) {
        const Prob &ap = args.probs[ic.p];
        ring_issue(ring, ap, ic.w.t, unit_id(ap, ic.w.slc, ic.u), lane);
        chain_next(args, warp, ic);
    }
    __syncthreads();
    // the counter is polled and advanced by a thread that issues no weight
    // copies (lane 1 of warp 0)
    constexpr int kSignal = 1;
    int rbuf = 0;
    int waited = 0;  // problems known complete
    for (int p = 0; p < args.count; ++p) {
        const Prob &a = args.probs[p];
        const int first = chain_first(args, p);
        const bool mine = first < a.items;
        // the outlier column indices are part of the packed layer: load them
        // before the wait
        const XRange xr = x_range(a, 0, 1, 1);
        XIdx xi;
        if (mine) load_x_idx(a, xr, 1, xi);
        // every CTA has finished the problems before p's stage (their y may
        // be this x); the acquire, then the CTA barrier, order the x loads
        // after it
        const int need = args.need[p];
        if (need > waited) {
            if (threadIdx.x == kSignal && !s_abort &&
                !counter_wait(args.done, (unsigned int)need * gridDim.x)) {
                s_abort = 1;
                atomicOr(&g_device_error, 1u);
            }
            __syncthreads();
            waited = need;
        }
        if (mine) {
            stage_x<1, true>(a, st, xr, xi);
            __syncthreads();
            for (int item = first; item < a.items; item += gridDim.x) {
                const ChainWork cw = chain_work(a, item, warp);
                const bool active = cw.t < a.T;
                const int nunits = active ? cw.slc.nsg + cw.slc.nob : 0;
                float yacc = 0.f;
                for (int u = 0; u < nunits; ++u) {
                    const uint8_t *stage = ring_acquire(ring, lane);
                    if (stage) compute_unit<1>(a, stage, lane, st, xr, unit_id(a, cw.slc, u), &yacc);
                    ring_release(ring);
                    if (ic.p < args.count) {
                        const Prob &ap = args.probs[ic.p];
                        ring_issue(ring, ap, ic.w.t, unit_id(ap, ic.w.slc, ic.u), lane);
                        chain_next(args, warp, ic);
                    }
                }
                float tot = yacc;
                if (a.ppc > 1) {
                    // the ppc warps of one tile meet on their own barrier (ids 1..tpc)
                    float *red = st.red + (size_t)rbuf * kPersistWarps * 32;
                    red[warp * 32 + lane] = yacc;
                    named_sync(1 + cw.tl, 32 * a.ppc);
                    if (cw.sl == 0) {
                        tot = 0.f;
                        for (int s2 = 0; s2 < a.ppc; ++s2) tot += red[(cw.tl * a.ppc + s2) * 32 + lane];
                    }
                    rbuf ^= 1;
                }
                if (cw.sl == 0 && active) store_y(a, cw.t, lane, 0, tot);
            }
        }
        // this CTA's rows of problem p are stored: count it done (a release,
        // after the CTA barrier, covers every warp's stores)
        __syncthreads();
        if (threadIdx.x == kSignal) red_release_gpu_add(args.done, 1u);
    }
    ring_drain(ring);
}

// ---------------------------------------------------------------- host planning

constexpr size_t kSmPerSm = 228 * 1024;  // shared memory of one SM
constexpr size_t kCtaReserve = 1024;     // per-CTA shared memory the system reserves
constexpr int kMaxDepth = 4;
// Ring stages a warp issues before it waits on the previous grid.  All of
// them would queue x's loads behind the whole of this SM's weights (x can
// only be read after the wait), so the decode could not start before the
// stream had landed; one stage per warp (about 75 KB per SM) covers the wait.
constexpr int kPreStages = 1;


int64_t tile_bytes(const Geometry &g) {
    return (int64_t)g.S * kSgBytes + (int64_t)g.O8 * kOctBytes;
}

int max_share(int total, int parts_per, int cl, int P) {
    int mx = 0;
    for (int c = 0; c < cl; ++c) {
        const int b = (int)(((int64_t)total * c * parts_per) / P);
        const int e = (int)(((int64_t)total * (c + 1) * parts_per) / P);
        if (e - b > mx) mx = e - b;
    }
    return mx;
}

// Deepest ring that fits `budget` with the x stage of `sm` (0 if none fits).
int fit_depth(int MB, int nw, Smem sm, size_t budget) {
    for (int d = kMaxDepth; d >= 1; --d) {
        sm.depth = d;
        if (stage_bytes(MB, nw, sm) <= budget) return d;
    }
    return 0;
}

// Cluster kernel: depth for two CTAs per SM if that leaves >= 2 stages per
// warp, else the deepest ring of one CTA.
int choose_depth(int MB, const Smem &sm, const DeviceInfo &dev) {
    const int d2 = fit_depth(MB, kClusterWarps, sm, kSmPerSm / 2 - kCtaReserve);
    if (d2 >= 2 || (d2 >= 1 && MB == 1 && fit_depth(MB, kClusterWarps, sm, dev.smem_optin) < 2))
        return d2;
    return fit_depth(MB, kClusterWarps, sm, dev.smem_optin);
}

int ctas_per_sm(int MB, const Smem &sm) {
    const int per = (int)(kSmPerSm / (stage_bytes(MB, kClusterWarps, sm) + kCtaReserve));
    const int reg_cap = MB == 1 ? 2 : 1;
    return per < 1 ? 1 : (per > reg_cap ? reg_cap : per);
}

struct ClusterPlan {
    int ppc, tpc, cl;
    Smem sm;
    unsigned grid;
    double cost;
};

// Clusters of `cl` CTAs of `smem` bytes each that the device runs at once.
// Clusters are placed within one GPC, so this can be well below
// sm_count * CTAs per SM / cl; a launch with more clusters runs a second
// wave.  Cached per device and shape (0: the shape cannot run).
template <int MB>
int cluster_capacity(int cl, size_t smem, const DeviceInfo &dev) {
    struct Entry {
        int device, cl;
        size_t smem;
        int cap;
    };
    static std::mutex mu;
    static Entry cache[256];
    static int n = 0;
    static bool done[64];
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (cache[i].device == dev.device && cache[i].cl == cl && cache[i].smem == smem) return cache[i].cap;
    int cap = 0;
    if (prepare_kernel(gemv_cluster_kernel<MB>, done, dev) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(cl * dev.sm_count), 1, 1);
        cfg.blockDim = dim3(kClusterWarps * 32, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = (unsigned)cl;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&cap, gemv_cluster_kernel<MB>, &cfg) != cudaSuccess) {
            cap = 0;
            (void)cudaGetLastError();
        }
    }
    if (n < 256) cache[n++] = Entry{dev.device, cl, smem, cap};
    return cap;
}

// Cluster kernel: slices per tile P = ppc * cl and tiles per CTA from a simple
// model -- waves of CTAs (of clusters, by the device's cluster capacity)
// times the bytes of the largest slice, plus a cost per CTA start and per
// reduction level.
template <int MB>
bool plan_cluster(const Geometry &g, const DeviceInfo &dev, ClusterPlan *out) {
    const int U = units_of(g);
    const int OB = U - g.S;
    bool found = false;
    out->cost = 1e300;
    for (int cl = 1; cl <= 8; ++cl) {
        for (int ppc = 1; ppc <= kClusterWarps; ++ppc) {
            const int P = ppc * cl;
            if (P > 1 && P > U) continue;
            const int tpc = kClusterWarps / ppc;
            Smem sm;
            sm.xg = 8 * max_share(g.S, ppc, cl, P);
            sm.xo = 8 * kOB * max_share(OB, ppc, cl, P);
            sm.tpc = tpc;
            sm.depth = choose_depth(MB, sm, dev);
            if (sm.depth == 0) continue;
            const int64_t ctas = cdiv(g.T, tpc) * cl;
            int64_t waves = cdiv(ctas, (int64_t)dev.sm_count * ctas_per_sm(MB, sm));
            if (cl > 1) {
                const int cap = cluster_capacity<MB>(cl, stage_bytes(MB, kClusterWarps, sm), dev);
                if (cap <= 0) continue;
                waves = cdiv(ctas / cl, cap);
            }
            const int64_t slice = cdiv(g.S, P) * kSgBytes + cdiv(OB, P) * kOB * kOctBytes;
            const double cost = (double)waves * (double)(slice + 8192) +
                                (ppc > 1 ? 256.0 * ppc : 0.0) + (cl > 1 ? 4096.0 + 512.0 * cl : 0.0);
            if (cost < out->cost) {
                found = true;
                out->cost = cost;
                out->ppc = ppc;
                out->tpc = tpc;
                out->cl = cl;
                out->sm = sm;
                out->grid = (unsigned)ctas;
            }
        }
    }
    return found;
}

// Persistent kernel: item = tpc tiles x ppc slices, ppc a power of two <= 16.
// Among the shapes whose item stays within twice `target` bytes (so that each
// CTA walks several items), take the one whose slices are most even -- the
// warps of a tile meet on a barrier at the end of an item -- and, on a tie,
// the fewest slices (more warps own whole tiles: no reduction at all).
void item_shape(const Geometry &g, int64_t target, int *ppc, int *tpc) {
    const int OB = (int)cdiv(g.O8, kOB);
    const int U = g.S + OB;
    const double tb = (double)tile_bytes(g);
    int best_p = 0;
    double best_eff = -1.0;
    for (int p = 1; p <= kPersistWarps; p *= 2) {
        if (p > 1 && p > U) break;
        if ((double)(kPersistWarps / p) * tb > 2.0 * (double)target && p < kPersistWarps) continue;
        // slowest slice vs mean slice, in bytes
        const double mean = tb / p;
        const double mx = (double)cdiv(g.S, p) * kSgBytes + (double)cdiv(OB, p) * kOB * kOctBytes;
        const double eff = mean / mx;
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best_p = p;
        }
    }
    if (best_p == 0) best_p = kPersistWarps;
    *ppc = best_p;
    *tpc = kPersistWarps / best_p;
}

// Item byte target: about `per_cta` items per CTA, at least 64 KB.
int64_t item_target(int64_t total, int ncta, int per_cta) {
    const int64_t t = total / ((int64_t)ncta * per_cta);
    return t < 65536 ? 65536 : t;
}

// A CTA whose range crosses into another matrix restages x there, a few
// microseconds of its stream; the split counts each change as this many bytes.
constexpr int64_t kRestageBytes = 192 * 1024;

// Contiguous item ranges of about equal cost (bytes, plus kRestageBytes per
// matrix change): boundary c goes to the item edge nearest c / ncta of the
// total, so a CTA is off its share by at most half an item.
void split_ctas(PersistArgs &args, int count, int ncta, int items) {
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        const Prob &a = args.probs[i];
        total += (int64_t)a.T * tile_bytes(Geometry::of(a.n, a.k, a.n_o)) + (i > 0 ? kRestageBytes : 0);
    }
    int64_t acc = 0;
    int c = 1;
    args.cta_first[0] = 0;
    for (int i = 0; i < count && c < ncta; ++i) {
        const Prob &a = args.probs[i];
        const int64_t tb = tile_bytes(Geometry::of(a.n, a.k, a.n_o));
        for (int it = 0; it < a.items && c < ncta; ++it) {
            const int idx = args.item_start[i] + it;
            const int64_t cost = (int64_t)min(a.tpc, a.T - it * a.tpc) * tb +
                                 (it == 0 && i > 0 ? kRestageBytes : 0);
            // boundaries whose ideal position falls inside this item
            while (c < ncta && (acc + cost) * ncta >= total * (int64_t)c) {
                const int64_t before = total * (int64_t)c - acc * ncta;
                const int64_t after = (acc + cost) * ncta - total * (int64_t)c;
                args.cta_first[c] = (before < after && idx > args.cta_first[c - 1]) ? idx : idx + 1;
                ++c;
            }
            acc += cost;
        }
    }
    while (c <= ncta) args.cta_first[c++] = items;
}

// The persistent launch over the `count` problems filled in args.probs.
template <int MB>
spectra_status run_persistent(PersistArgs &args, int count, const DeviceInfo &dev, cudaStream_t s) {
    static bool done[64];
    Smem sm = {1, 0, 0, 0};
    int items = 0;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        const Prob &a = args.probs[i];
        total += (int64_t)a.T * tile_bytes(Geometry::of(a.n, a.k, a.n_o));
    }
    // items of a few per cent of a CTA's share: narrower items would split
    // tiles into more slices (idle warps on short tiles, a reduction per item)
    const int64_t target = item_target(total, dev.sm_count, 8);
    total = 0;
    for (int i = 0; i < count; ++i) {
        Prob &a = args.probs[i];
        const Geometry g = Geometry::of(a.n, a.k, a.n_o);
        item_shape(g, target, &a.ppc, &a.tpc);
        a.lgp = 0;
        while ((1 << a.lgp) < a.ppc) ++a.lgp;
        a.items = (int)cdiv(a.T, a.tpc);
        args.item_start[i] = items;
        items += a.items;
        sm.xg = max(sm.xg, 8 * a.S);
        sm.xo = max(sm.xo, 8 * kOB * (a.U - a.S));
    }
    args.item_start[count] = items;
    args.count = count;
    sm.depth = fit_depth(MB, kPersistWarps, sm, dev.smem_optin);
    if (sm.depth > 2) sm.depth = 2;  // 16 warps x 2 stages keep ~150 KB in flight per SM
    if (sm.depth == 0) return SPECTRA_ERR_SHAPE;
    args.sm = sm;
    args.pre = kPreStages;
    int ncta = dev.sm_count;
    if (ncta > kMaxCtas) ncta = kMaxCtas;
    if (ncta > items) ncta = items;
    split_ctas(args, count, ncta, items);
    cudaError_t e = prepare_kernel(gemv_persistent_kernel<MB>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    e = launch_kernel(gemv_persistent_kernel<MB>, args, (unsigned)ncta,
                      stage_bytes(MB, kPersistWarps, sm), kPersistWarps, 1, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

// Chain kernel: per problem the item shape (tpc tiles x ppc slices, tpc x
// ppc = 16) whose busiest warp holds the fewest units, items dealt round
// robin over `ncta` CTAs.
void chain_shape(const Geometry &g, int ncta, int *ppc, int *tpc) {
    const int U = g.S + (int)cdiv(g.O8, kOB);
    double best_cost = 1e300;
    for (int p = 1; p <= kPersistWarps; p *= 2) {
        const int tp = kPersistWarps / p;
        const int64_t items = cdiv(g.T, tp);
        const double cost = (double)cdiv(items, ncta) * (double)cdiv(U, p) + (p > 1 ? 0.02 * p : 0.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            *ppc = p;
            *tpc = tp;
        }
    }
}

spectra_status run_chain(ChainArgs &args, int count, void *ws, size_t ws_bytes, const DeviceInfo &dev,
                         cudaStream_t s) {
    const int ncta = dev.sm_count;
    if (ws_bytes < kChainWorkspace) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    Smem sm = {1, 0, 0, 0};
    for (int i = 0; i < count; ++i) {
        Prob &a = args.probs[i];
        const Geometry g = Geometry::of(a.n, a.k, a.n_o);
        chain_shape(g, ncta, &a.ppc, &a.tpc);
        a.lgp = 0;
        a.items = (int)cdiv(a.T, a.tpc);
        args.base[i] = (i > 0 && args.need[i] == args.need[i - 1]) ? args.base[i - 1] + args.probs[i - 1].items : 0;
        sm.xg = max(sm.xg, 8 * a.S);
        sm.xo = max(sm.xo, 8 * kOB * (a.U - a.S));
    }
    sm.depth = fit_depth(1, kPersistWarps, sm, dev.smem_optin);
    if (sm.depth > 2) sm.depth = 2;
    if (sm.depth == 0) return SPECTRA_ERR_SHAPE;
    args.sm = sm;
    args.count = count;
    args.done = static_cast<unsigned int *>(ws);
    const size_t smem = stage_bytes(1, kPersistWarps, sm);
    // the kernel also has a static shared word: raise the dynamic limit to
    // what this launch needs (the device maximum would leave no room for it)
    cudaError_t e = cudaFuncSetAttribute(gemv_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    // every CTA waits on the others, so all of them must be resident at once:
    // one CTA per SM, which the device must be able to hold
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_chain_kernel, kPersistWarps * 32,
                                                      smem) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (per_sm < 1) return SPECTRA_ERR_SHAPE;
    // the counter starts at zero in every launch
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    gemv_chain_kernel<<<(unsigned)ncta, kPersistWarps * 32, smem, s>>>(args);
    return cudaGetLastError() == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

template <int MB>
spectra_status run_cluster(const Prob &a0, const ClusterPlan &p, const DeviceInfo &dev,
                           cudaStream_t s) {
    static bool done[64];
    ClusterArgs args;
    args.p = a0;
    args.p.ppc = p.ppc;
    args.p.tpc = p.tpc;
    args.p.cl = p.cl;
    args.sm = p.sm;
    args.pre = kPreStages;
    cudaError_t e = prepare_kernel(gemv_cluster_kernel<MB>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    e = launch_kernel(gemv_cluster_kernel<MB>, args, p.grid, stage_bytes(MB, kClusterWarps, p.sm),
                      kClusterWarps, p.cl, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

// One matrix, MB batch rows: the persistent kernel when the matrix gives every
// SM several balanced items (large matrices), else the cluster kernel.
template <int MB>
spectra_status run_one(const Prob &a, const DeviceInfo &dev, cudaStream_t s) {
    const Geometry g = Geometry::of(a.n, a.k, a.n_o);
    const int64_t total = (int64_t)g.T * tile_bytes(g);
    int ppc, tpc;
    item_shape(g, item_target(total, dev.sm_count, 8), &ppc, &tpc);
    const int64_t items = cdiv(g.T, tpc);
    if (items >= 4LL * dev.sm_count && total >= (int64_t)dev.sm_count * 512 * 1024) {
        static std::mutex mu;
        static PersistArgs args;  // large: kept off the stack, guarded by the mutex
        std::lock_guard<std::mutex> lock(mu);
        args.probs[0] = a;
        return run_persistent<MB>(args, 1, dev, s);
    }
    ClusterPlan p;
    if (!plan_cluster<MB>(g, dev, &p)) return SPECTRA_ERR_SHAPE;
    return run_cluster<MB>(a, p, dev, s);
}

// One warp acquires the first stage of a one-stage weight ring that no copy
// ever fills: the ring's bounded wait gives up after its limit and raises
// this translation unit's error flag, exactly as in a matvec kernel.
__global__ void ring_wait_selftest_kernel() {
    __shared__ __align__(16) uint8_t stage[16];
    __shared__ __align__(8) uint64_t bar[1];
    const int lane = threadIdx.x & 31;
    Ring r;
    ring_init(r, stage, bar, 1, lane);
    (void)ring_acquire(r, lane);
    ring_release(r);
    ring_drain(r);
}

// A counter that no kernel ever increments.
__device__ unsigned int g_never_counted;

// One thread waits, as a chain CTA waits for the others, on a counter that
// never reaches its target: the bounded wait gives up and raises the flag.
__global__ void counter_wait_selftest_kernel() {
    if (threadIdx.x == 0 && !counter_wait(&g_never_counted, 1u)) atomicOr(&g_device_error, 1u);
}

}  // namespace

// This translation unit's error word (the matvec kernels), then the
// tensor-core kernel's (gemm_tc.cu).
spectra_status device_error(unsigned int *bits, cudaStream_t s) {
    unsigned int tc_bits = 0;
    const spectra_status st = tc_device_error(&tc_bits, s);
    if (st != SPECTRA_OK) return st;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    *bits = v | tc_bits;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                    s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
    }
    return SPECTRA_OK;
}

spectra_status launch_gemv(const spectra_layer &l, const uint16_t *x, int m, void *y, int ytype,
                           cudaStream_t s, const DeviceInfo &dev) {
    // 8 or more batch rows: a real dense contraction, on the tensor cores
    // (measured faster than the CUDA-core decode from 8 rows on)
    if (m >= 8) return launch_tc(l, x, m, y, ytype, s, dev);
    const Geometry g = Geometry::of(l.n, bulk_cols(l), l.n_outliers);
    int done = 0;
    while (done < m) {
        const int mc = (m - done) > 8 ? 8 : (m - done);
        const int MB = mc == 1 ? 1 : (mc == 2 ? 2 : (mc <= 4 ? 4 : 8));
        Prob a;
        void *yc = (ytype == SPECTRA_F32)
                       ? (void *)(reinterpret_cast<float *>(y) + (size_t)done * l.n)
                       : (void *)(reinterpret_cast<uint16_t *>(y) + (size_t)done * l.n);
        fill_prob(a, l, g, x + (size_t)done * l.k, mc, yc, ytype);
        spectra_status st;
        switch (MB) {
            case 1: st = run_one<1>(a, dev, s); break;
            case 2: st = run_one<2>(a, dev, s); break;
            case 4: st = run_one<4>(a, dev, s); break;
            default: st = run_one<8>(a, dev, s); break;
        }
        if (st != SPECTRA_OK) return st;
        done += mc;
    }
    return SPECTRA_OK;
}

spectra_status launch_gemv_batched(const spectra_layer *layers, const uint16_t *const *xs,
                                   void *const *ys, int count, int ytype, cudaStream_t s,
                                   const DeviceInfo &dev) {
    static std::mutex mu;
    static PersistArgs args;  // large: kept off the stack, guarded by the mutex
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < count; ++i) {
        const Geometry g = Geometry::of(layers[i].n, bulk_cols(layers[i]), layers[i].n_outliers);
        fill_prob(args.probs[i], layers[i], g, xs[i], 1, ys[i], ytype);
    }
    // one matrix: spectra_gemv's choice of kernel (the cluster kernel unless
    // the matrix is large)
    if (count == 1) return run_one<1>(args.probs[0], dev, s);
    return run_persistent<1>(args, count, dev, s);
}

spectra_status launch_gemv_chain(const spectra_layer *layers, const uint16_t *const *xs,
                                 void *const *ys, int count, int ytype, const int32_t *stage,
                                 void *ws, size_t ws_bytes, cudaStream_t s, const DeviceInfo &dev) {
    static std::mutex mu;
    static ChainArgs args;  // large: kept off the stack, guarded by the mutex
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < count; ++i) {
        const Geometry g = Geometry::of(layers[i].n, bulk_cols(layers[i]), layers[i].n_outliers);
        fill_prob(args.probs[i], layers[i], g, xs[i], 1, ys[i], ytype);
        // no stages: every problem waits for all earlier ones
        args.need[i] = (uint16_t)((stage && i > 0 && stage[i] == stage[i - 1]) ? args.need[i - 1] : i);
    }
    return run_chain(args, count, ws, ws_bytes, dev, s);
}

size_t gemv_chain_workspace_bytes() { return kChainWorkspace; }

spectra_status launch_wait_selftest(int kind, cudaStream_t s) {
    if (kind == 0)
        ring_wait_selftest_kernel<<<1, 32, 0, s>>>();
    else if (kind == 1)
        counter_wait_selftest_kernel<<<1, 32, 0, s>>>();
    else
        return SPECTRA_ERR_INVALID_ARG;
    return cudaGetLastError() == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

}  // namespace spectra
