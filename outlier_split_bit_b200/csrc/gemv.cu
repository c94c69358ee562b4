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
// launch once all of its CTAs run, issues its first D units of (constant)
// weights, and only then waits for the previous grid before it reads x or
// writes y.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace spectra {
namespace {

constexpr int kClusterWarps = 8;               // warps per CTA of the cluster kernel
constexpr int kPersistWarps = 16;              // warps per CTA of the persistent kernel
constexpr int kOB = 8;                         // outlier octets per unit
constexpr int kSgBytes = 8 * 512 + 512 + 128;  // codes + scales + zeros of a warp per super-group
constexpr int kOctBytes = 512;                 // outlier bytes of a warp per octet
constexpr int kStageBytes = kSgBytes;          // one ring stage (16-byte multiple)
constexpr uint32_t kSpinLimit = 1u << 12;      // try_wait rounds before a wait gives up
constexpr uint32_t kSuspendNs = 500000;        // per-round suspend hint: the limit is ~2 s
constexpr int kMaxCtas = 320;                  // persistent grid bound (2 x SMs of a B200 + margin)

// Set (bit 0) when a bounded wait in a kernel gave up; read and cleared by
// spectra_device_status().
__device__ unsigned int g_device_error;

// One matvec problem as the kernels see it.
struct Prob {
    const uint4 *codes;
    const uint4 *scales;
    const uint32_t *zeros;
    const uint4 *outw;
    const int32_t *oidx;
    const uint16_t *x;
    void *y;
    int n, k, m, G, S, O8, n_o, T;
    int U;         // units per tile
    int ppc, tpc;  // slices per tile, tiles per CTA item
    int cl;        // CTAs per cluster (cluster kernel)
    int ytype;
    int items;     // ceil(T / tpc)
};

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
};

// Parameters of the persistent kernel, passed by value (kernel parameter space).
struct PersistArgs {
    Smem sm;
    int count;                      // problems
    int item_start[kMaxBatch + 1];  // first item of each problem
    int cta_first[kMaxCtas + 1];    // first item of each CTA
    Prob probs[kMaxBatch];
};
static_assert(sizeof(PersistArgs) <= 32760, "kernel parameter space");

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Barrier among the `threads` threads (a multiple of 32) that use barrier `id`.
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// floor(total * s / P); total * s stays far below 2^31 (total <= a few
// thousand units, s <= 16), so 32-bit arithmetic is exact.
__device__ __forceinline__ int split_at(int total, int s, int P) {
    return (int)((unsigned)(total * s) / (unsigned)P);
}


__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Wait for phase `parity` of an mbarrier; gives up after kSpinLimit rounds.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t ok;
        // the thread sleeps until the phase completes or the hint expires,
        // so waiting warps leave the issue slots to the computing ones
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(kSuspendNs)
            : "memory");
        if (ok) return true;
    }
    return false;
}

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

// Stage x for a unit range: bulk groups as BF16 pairs in the decoder's order
// with their FP32 sums X_g (column order), and the BF16 pairs of the outlier
// slots, gathered through the index list.
template <int MB>
__device__ void stage_x(const Prob &a, const Stage<MB> &st, const XRange &xr) {
    const int nth = blockDim.x;
    const int ng = xr.g1 - xr.g0;
    for (int c = threadIdx.x; c < ng * MB; c += nth) {
        const int gl = c / MB, m = c - gl * MB;
        const int g = xr.g0 + gl;
        uint32_t *dst = st.xs + (size_t)gl * 16 * MB + m;
        float sum = 0.f;
        if (g < a.G && m < a.m) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.k + 32 * g);
            uint4 v[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) v[w] = src[w];
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
    // outlier slots as BF16 pairs: 8 pairs per thread in flight
    const int np = (xr.j1 - xr.j0) / 2;
    for (int base = 0; base < np * MB; base += 8 * nth) {
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
                const uint32_t lo = (i0[i] >= 0 && mv) ? a.x[(size_t)m * a.k + i0[i]] : 0u;
                const uint32_t hi = (i1[i] >= 0 && mv) ? a.x[(size_t)m * a.k + i1[i]] : 0u;
                st.xo[c] = lo | (hi << 16);
            }
        }
    }
}

// ---------------------------------------------------------------- units

// Copies of unit u of tile t into ring stage `dst`.  Called by one lane.
__device__ __forceinline__ void issue_unit(const Prob &a, int t, int u, uint32_t dst,
                                           uint32_t bar) {
    if (u < a.S) {
        const int ng = min(8, a.G - 8 * u);
        const uint32_t cb = (uint32_t)ng * 512u;
        mbar_expect_tx(bar, cb + 512u + 128u);
        bulk_g2s(dst, a.codes + ((size_t)t * a.G + 8 * u) * 32, cb, bar);
        bulk_g2s(dst + 4096u, a.scales + ((size_t)t * a.S + u) * 32, 512u, bar);
        bulk_g2s(dst + 4608u, a.zeros + ((size_t)t * a.S + u) * 32, 128u, bar);
    } else {
        const int oc = (u - a.S) * kOB;
        const uint32_t b = (uint32_t)min(kOB, a.O8 - oc) * 512u;
        mbar_expect_tx(bar, b);
        bulk_g2s(dst, a.outw + ((size_t)t * a.O8 + oc) * 32, b, bar);
    }
}

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

// BF16 pair (128 + c_s, 128 + c_{s+4}) of nibbles s and s + 4 of a word.
template <int sh>
__device__ __forceinline__ uint32_t code_pair(uint32_t w) {
    return ((w >> (4 * sh)) & 0x000F000Fu) | 0x43004300u;
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

__device__ __forceinline__ void store_y(const Prob &a, int t, int lane, int m, float v) {
    const int row = 32 * t + lane;
    if (row < a.n && m < a.m) {
        if (a.ytype == SPECTRA_F32)
            reinterpret_cast<float *>(a.y)[(size_t)m * a.n + row] = v;
        else
            reinterpret_cast<__nv_bfloat16 *>(a.y)[(size_t)m * a.n + row] = __float2bfloat16_rn(v);
    }
}

// Per-warp ring of D stages: units are consumed in the order they were issued.
struct Ring {
    uint8_t *base;
    uint32_t base_s, bar_s;
    int D;
    int consumed, issued;
    bool ok;
    int failed_at;
};

__device__ __forceinline__ void ring_init(Ring &r, uint8_t *base, uint64_t *bars, int D, int lane) {
    r.base = base;
    r.base_s = smem_u32(base);
    r.bar_s = smem_u32(bars);
    r.D = D;
    r.consumed = r.issued = 0;
    r.ok = true;
    r.failed_at = 0;
    if (lane == 0) {
        for (int d = 0; d < D; ++d) mbar_init(r.bar_s + 8u * d, 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
}

__device__ __forceinline__ void ring_issue(Ring &r, const Prob &a, int t, int u, int lane) {
    const int d = r.issued % r.D;
    if (r.ok && lane == 0)
        issue_unit(a, t, u, r.base_s + (uint32_t)d * kStageBytes, r.bar_s + 8u * d);
    if (r.ok) ++r.issued;
}

// Wait for the next stage to fill; returns its address (nullptr after a failure).
__device__ __forceinline__ const uint8_t *ring_acquire(Ring &r, int lane) {
    const int d = r.consumed % r.D;
    if (r.ok && !mbar_wait(r.bar_s + 8u * d, (uint32_t)(r.consumed / r.D) & 1u)) {
        r.ok = false;
        r.failed_at = r.consumed;
        if (lane == 0) atomicOr(&g_device_error, 1u);
    }
    return r.ok ? r.base + (size_t)d * kStageBytes : nullptr;
}

__device__ __forceinline__ void ring_release(Ring &r) {
    __syncwarp();
    if (r.ok) ++r.consumed;
}

// After a failed wait, let the copies already in flight land before the CTA
// releases its shared memory (bounded as well).
__device__ __forceinline__ void ring_drain(const Ring &r) {
    if (r.ok) return;
    for (int n = r.failed_at; n < r.issued; ++n)
        mbar_wait(r.bar_s + 8u * (n % r.D), (uint32_t)(n / r.D) & 1u);
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
    int next = 0;
    for (; next < nunits && next < ring.D; ++next) ring_issue(ring, a, t, unit_id(a, slc, next), lane);
    pdl_wait();
    stage_x<MB>(a, st, xr);
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

// Move the cursor to the first unit of `c.item` or of a later item of this warp.
__device__ __forceinline__ void cursor_load(const PersistArgs &args, int it1, int warp, Cursor &c) {
    while (c.item < it1) {
        c.p = prob_of(args, c.item);
        const Prob &a = args.probs[c.p];
        const int blk = c.item - args.item_start[c.p];
        const int tl = warp / a.ppc;
        c.t = blk * a.tpc + tl;
        if (c.t < a.T) {
            c.sl = slice_of(a, warp - tl * a.ppc, a.ppc);
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
    cursor_load(args, it1, warp, ic);
    for (int d = 0; d < ring.D && ic.item < it1; ++d) {
        cursor_issue(args, ring, ic, lane);
        cursor_next(args, it1, warp, ic);
    }
    pdl_wait();

    int cur_p = -1;
    int rbuf = 0;
    XRange xr = {0, 0, 0, 0};
    for (int item = it0; item < it1; ++item) {
        const int p = prob_of(args, item);
        const Prob &a = args.probs[p];
        if (p != cur_p) {
            // every warp is done with the previous x (the branch is CTA-uniform)
            __syncthreads();
            xr = x_range(a, 0, 1, 1);
            stage_x<MB>(a, st, xr);
            __syncthreads();
            cur_p = p;
        }
        const int blk = item - args.item_start[p];
        const int tl = warp / a.ppc, sl = warp - tl * a.ppc;
        const int t = blk * a.tpc + tl;
        const bool active = t < a.T;
        const Slice slc = slice_of(a, sl, a.ppc);
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

// ---------------------------------------------------------------- host planning

constexpr size_t kSmPerSm = 228 * 1024;  // shared memory of one SM
constexpr size_t kCtaReserve = 1024;     // per-CTA shared memory the system reserves
constexpr int kMaxDepth = 4;

int units_of(const Geometry &g) { return g.S + (int)cdiv(g.O8, kOB); }

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

// Cluster kernel: slices per tile P = ppc * cl and tiles per CTA from a simple
// model -- waves of CTAs times the bytes of the largest slice, plus a cost per
// CTA start and per reduction level.
bool plan_cluster(const Geometry &g, int MB, const DeviceInfo &dev, ClusterPlan *out) {
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
            const int64_t waves = cdiv(ctas, (int64_t)dev.sm_count * ctas_per_sm(MB, sm));
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

// Item byte target: about 8 items per CTA, at least 64 KB.
int64_t item_target(int64_t total, int ncta) {
    const int64_t t = total / ((int64_t)ncta * 8);
    return t < 65536 ? 65536 : t;
}

void fill_prob(Prob &a, const spectra_layer &l, const Geometry &g, const uint16_t *x, int mc,
               void *y, int ytype) {
    a.codes = reinterpret_cast<const uint4 *>(l.codes);
    a.scales = reinterpret_cast<const uint4 *>(l.scales);
    a.zeros = l.zeros;
    a.outw = reinterpret_cast<const uint4 *>(l.outlier_w);
    a.oidx = l.outlier_idx;
    a.x = x;
    a.y = y;
    a.n = l.n;
    a.k = l.k;
    a.m = mc;
    a.G = g.G;
    a.S = g.S;
    a.O8 = g.O8;
    a.n_o = g.n_o;
    a.T = g.T;
    a.U = units_of(g);
    a.ppc = 1;
    a.tpc = 1;
    a.cl = 1;
    a.ytype = ytype;
    a.items = 0;
}

std::mutex g_attr_mu;

// Raise the dynamic shared-memory limit of one kernel, once per device.
template <typename K>
cudaError_t prepare_kernel(K kernel, bool *done, const DeviceInfo &dev) {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (dev.device >= 0 && dev.device < 64 && done[dev.device]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dev.smem_optin);
    if (e == cudaSuccess && dev.device >= 0 && dev.device < 64) done[dev.device] = true;
    return e;
}

template <typename K, typename A>
cudaError_t launch_kernel(K kernel, const A &args, unsigned grid, size_t smem, int nw, int cl,
                          cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(nw * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cl > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = cl;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, args);
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
    const int64_t target = item_target(total, dev.sm_count);
    total = 0;
    for (int i = 0; i < count; ++i) {
        Prob &a = args.probs[i];
        const Geometry g = Geometry::of(a.n, a.k, a.n_o);
        item_shape(g, target, &a.ppc, &a.tpc);
        a.items = (int)cdiv(a.T, a.tpc);
        args.item_start[i] = items;
        items += a.items;
        total += (int64_t)a.T * tile_bytes(g);
        sm.xg = max(sm.xg, 8 * a.S);
        sm.xo = max(sm.xo, 8 * kOB * (a.U - a.S));
    }
    args.item_start[count] = items;
    args.count = count;
    sm.depth = fit_depth(MB, kPersistWarps, sm, dev.smem_optin);
    if (sm.depth > 2) sm.depth = 2;  // 16 warps x 2 stages keep ~150 KB in flight per SM
    if (sm.depth == 0) return SPECTRA_ERR_SHAPE;
    args.sm = sm;
    int ncta = dev.sm_count;
    if (ncta > kMaxCtas) ncta = kMaxCtas;
    if (ncta > items) ncta = items;
    // contiguous item ranges of about equal bytes
    int64_t acc = 0;
    int c = 1;
    args.cta_first[0] = 0;
    for (int i = 0; i < count && c < ncta; ++i) {
        const Prob &a = args.probs[i];
        const Geometry g = Geometry::of(a.n, a.k, a.n_o);
        for (int it = 0; it < a.items && c < ncta; ++it) {
            const int tiles = min(a.tpc, a.T - it * a.tpc);
            acc += (int64_t)tiles * tile_bytes(g);
            while (c < ncta && acc * ncta >= total * (int64_t)c)
                args.cta_first[c++] = args.item_start[i] + it + 1;
        }
    }
    while (c <= ncta) args.cta_first[c++] = items;
    cudaError_t e = prepare_kernel(gemv_persistent_kernel<MB>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    e = launch_kernel(gemv_persistent_kernel<MB>, args, (unsigned)ncta,
                      stage_bytes(MB, kPersistWarps, sm), kPersistWarps, 1, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
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
    item_shape(g, item_target(total, dev.sm_count), &ppc, &tpc);
    const int64_t items = cdiv(g.T, tpc);
    if (items >= 4LL * dev.sm_count && total >= (int64_t)dev.sm_count * 512 * 1024) {
        static std::mutex mu;
        static PersistArgs args;  // large: kept off the stack, guarded by the mutex
        std::lock_guard<std::mutex> lock(mu);
        args.probs[0] = a;
        return run_persistent<MB>(args, 1, dev, s);
    }
    ClusterPlan p;
    if (!plan_cluster(g, MB, dev, &p)) return SPECTRA_ERR_SHAPE;
    return run_cluster<MB>(a, p, dev, s);
}

// ---------------------------------------------------------------- tensor-core path (M = 16..32)
//
// y[m][n] for 16 <= m_rows <= 32 (MB = 16 or 32 batch rows) on the fifth-
// generation tensor cores.  A CTA owns blocks of 128 rows (4 tiles; TMEM
// lane = row) and streams their units (super-groups, outlier batches) with
// three kinds of warps:
//
//  * two sets of four compute warps.  Set j takes every second unit of the
//    block; warp 4j + r owns tile r (rows 32r..32r+31) and keeps its own
//    cp.async.bulk ring of that tile's units.  Per group of 32 columns it
//    writes the exact integer weights c - z as a BF16 A operand (128 rows x
//    32 columns) into a TMEM buffer, and later reads back that group's FP32
//    product D = (c - z) x from TMEM and adds s * D to its rows' sums.  The
//    outlier columns enter the same way with their BF16 weights and s = 1.
//  * one MMA warp whose elected lane issues two tcgen05.mma kind::f16
//    (M = 128, N = MB, K = 16) per group and commits them to the group's
//    mbarrier.
//
// The products are exact: c - z is an integer in [-15, 15] and x is BF16, so
// each product has at most 12 significant bits; D holds FP32 sums of 32 of
// them and the per-group scale is applied in FP32 afterwards, as in the
// CUDA-core path.  The B operand (x) of each unit is staged by the set's
// threads in shared memory in the K-major canonical layout (8 x 16-byte core
// matrices, K halves 128 B apart, 8-row groups 256 B apart), in the order
// the decoder pairs the codes: the two BF16 halves of TMEM column 4w + s are
// columns 8w + s and 8w + s + 4 of the group.
//
// Handshakes, per set and TMEM buffer b (kTcP buffers, used round robin):
// full[b] (128 compute threads arrive after their TMEM stores and x writes)
// -> MMA issue -> done[b] (tcgen05.commit) -> compute threads read D[b].
// A buffer is rewritten only after its previous D was read, so the MMA that
// read its A has completed.  Every wait is bounded; a timeout raises the
// device error bit and turns the remaining waits into no-ops.
constexpr int kTcSets = 2;
constexpr int kTcComputeWarps = 4 * kTcSets;
constexpr int kTcWarps = kTcComputeWarps + 1;  // + the MMA warp
constexpr int kTcTmemCols = 512;

template <int MB>
struct TcCfg {
    static constexpr int P = MB == 32 ? 5 : 8;       // TMEM buffers per set
    static constexpr int L = P - 1;                  // groups produced ahead of the one read back
    static constexpr int DCOL = kTcSets * P * 16;    // A buffers at [0, DCOL), D after
    static constexpr int XBYTES = 256 * MB * 2;      // x image of one super-group
    static constexpr int KSTEP = MB * 32;            // bytes of one 16-column K step of x
    static_assert(DCOL + kTcSets * P * MB <= kTcTmemCols, "TMEM budget");
    static_assert(DCOL % 32 == 0, "D alignment");
};

struct TcArgs {
    Prob p;
    int depth;  // ring stages per compute warp
    int nblk;   // 128-row blocks
};

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    // start address, leading and stride byte offsets (all >> 4), version 1,
    // base offset 0, no swizzle
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

template <int MB>
__device__ __forceinline__ uint32_t bf16_idesc() {
    // D = F32 (bits 4-5 = 1), A = B = BF16 (format 1 at bits 7 and 10), both
    // K-major, N = MB (>> 3 at bit 17), M = 128 (>> 4 at bit 24)
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MB >> 3) << 17) | (8u << 24);
}

// Groups (of 32 columns) in unit u: a super-group has up to 8, an outlier
// batch one per four octets.
__device__ __forceinline__ int tc_groups(const Prob &a, int u) {
    if (u < a.S) return min(8, a.G - 8 * u);
    return (min(kOB, a.O8 - kOB * (u - a.S)) + 3) >> 2;
}

// Unit of local index lu of a CTA whose split is [sg0, sg0 + nsg) super-groups
// and [ob0, ...) outlier batches.
__device__ __forceinline__ int tc_unit(const Prob &a, int sg0, int nsg, int ob0, int lu) {
    return lu < nsg ? sg0 + lu : a.S + ob0 + (lu - nsg);
}

// Shared state of a CTA that turns every later wait into a no-op once one
// has timed out.
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

constexpr uint64_t kTcWaitNs = 1000000000ull;  // a wait gives up after one second

__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int *abort) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if ((i & 255u) == 0u) {
            if (*abort) return false;
            const uint64_t now = global_ns();
            if (i == 0) t0 = now;
            else if (now - t0 > kTcWaitNs) break;
        }
    }
    *abort = 1;
    atomicOr(&g_device_error, 1u);
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// x of one unit for one thread of a set (tid in [0, 128)), loaded one unit
// ahead into registers.  Super-group: MB/4 chunks of 8 consecutive columns
// (chunk c = tid + 128 i: row m = c % MB, word W = c / MB).  Outlier batch:
// MB/16 chunks of 8 gathered columns (row m = c % MB, octet c / MB).
template <int MB>
struct TcX {
    uint4 v[MB / 4];
};

template <int MB>
__device__ __forceinline__ void tc_load_x(const Prob &a, int u, int tid, TcX<MB> &xp) {
    if (u < a.S) {
        // only valid addresses: batch rows past m_rows read row m_rows - 1 and
        // chunks past the super-group's end read its last chunk (their
        // products land in D columns, or groups, that are never used)
        const int nw = 4 * min(8, a.G - 8 * u);
#pragma unroll
        for (int i = 0; i < MB / 4; ++i) {
            const int c = tid + 128 * i, m = min(c % MB, a.m - 1), W = min(c / MB, nw - 1);
            xp.v[i] = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.k + 256 * u + 8 * W));
        }
    } else {
        const int ob = u - a.S;
#pragma unroll
        for (int i = 0; i < MB / 16; ++i) {
            const int c = tid + 128 * i, m = c % MB, o = c / MB;
            const int j0 = 8 * (kOB * ob + o);
            int ix[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) ix[e] = (j0 + e < a.n_o) ? __ldg(a.oidx + j0 + e) : -1;
            // padding slots read column 0 and are zeroed when stored
            const uint16_t *row = a.x + (size_t)min(m, a.m - 1) * a.k;
            uint32_t h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = (uint32_t)__ldg(row + max(ix[e], 0));
            xp.v[i] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                 h[6] | (h[7] << 16));
        }
    }
}

// Write the prefetched x of unit u as the B image: chunk W goes to K step
// W / 2, core-matrix column W % 2.  Super-group chunks are reordered to
// (x0, x4, x1, x5, x2, x6, x3, x7), the decoder's pairing.
template <int MB>
__device__ __forceinline__ void tc_store_x(const Prob &a, int u, int tid, const TcX<MB> &xp,
                                           uint8_t *xb) {
    if (u < a.S) {
#pragma unroll
        for (int i = 0; i < MB / 4; ++i) {
            const int c = tid + 128 * i, m = c % MB, W = c / MB;
            const uint4 v = xp.v[i];
            const uint4 p = make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                                       __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632));
            *reinterpret_cast<uint4 *>(xb + (W >> 1) * TcCfg<MB>::KSTEP + (m >> 3) * 256 +
                                       (W & 1) * 128 + (m & 7) * 16) = p;
        }
    } else {
#pragma unroll
        for (int i = 0; i < MB / 16; ++i) {
            const int c = tid + 128 * i, m = c % MB, o = c / MB;
            const uint4 v = xp.v[i];
            // slots past n_o are padding: their x is zero
            const int nv = a.n_o - 8 * (kOB * (u - a.S) + o);
            const uint32_t k0 = nv >= 2 ? 0xFFFFFFFFu : (nv == 1 ? 0x0000FFFFu : 0u);
            const uint32_t k1 = nv >= 4 ? 0xFFFFFFFFu : (nv == 3 ? 0x0000FFFFu : 0u);
            const uint32_t k2 = nv >= 6 ? 0xFFFFFFFFu : (nv == 5 ? 0x0000FFFFu : 0u);
            const uint32_t k3 = nv >= 8 ? 0xFFFFFFFFu : (nv == 7 ? 0x0000FFFFu : 0u);
            *reinterpret_cast<uint4 *>(xb + (o >> 1) * TcCfg<MB>::KSTEP + (m >> 3) * 256 +
                                       (o & 1) * 128 + (m & 7) * 16) =
                make_uint4(v.x & k0, v.y & k1, v.z & k2, v.w & k3);
        }
    }
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

template <int MB>
__device__ __forceinline__ void tmem_ld_d(uint32_t taddr, float *d) {
    uint32_t r[MB];
    if constexpr (MB == 32) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
            "%28, %29, %30, %31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
              "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
              "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
              "=r"(r[31])
            : "r"(taddr)
            : "memory");
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr)
            : "memory");
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < MB; ++i) d[i] = __uint_as_float(r[i]);
}

// The A operand of group g of a unit for one row (lane): 16 TMEM columns of
// BF16 pairs, and the group's scale.
__device__ __forceinline__ float tc_build_a(const Prob &a, int u, int g, const uint8_t *stage,
                                            int lane, uint32_t *av) {
    if (!stage) {
#pragma unroll
        for (int i = 0; i < 16; ++i) av[i] = 0u;
        return 0.f;
    }
    if (u < a.S) {
        const uint4 q = *reinterpret_cast<const uint4 *>(stage + g * 512 + lane * 16);
        const uint32_t sw = *reinterpret_cast<const uint32_t *>(stage + 4096 + lane * 16 + (g >> 1) * 4);
        const uint32_t zw = *reinterpret_cast<const uint32_t *>(stage + 4608 + lane * 4);
        const uint32_t z = (zw >> (4 * g)) & 0xFu;
        const uint32_t zz = (0x4300u | z) * 0x00010001u;  // BF16 pair (128 + z, 128 + z)
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            av[4 * w + 0] = bf16x2_sub(code_pair<0>(wv[w]), zz);
            av[4 * w + 1] = bf16x2_sub(code_pair<1>(wv[w]), zz);
            av[4 * w + 2] = bf16x2_sub(code_pair<2>(wv[w]), zz);
            av[4 * w + 3] = bf16x2_sub(code_pair<3>(wv[w]), zz);
        }
        return __half2float(__ushort_as_half((unsigned short)((g & 1) ? (sw >> 16) : (sw & 0xFFFFu))));
    }
    const int nv = min(kOB, a.O8 - kOB * (u - a.S));
#pragma unroll
    for (int o = 0; o < 4; ++o) {
        uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
        if (4 * g + o < nv) w4 = *reinterpret_cast<const uint4 *>(stage + (4 * g + o) * 512 + lane * 16);
        av[4 * o + 0] = w4.x;
        av[4 * o + 1] = w4.y;
        av[4 * o + 2] = w4.z;
        av[4 * o + 3] = w4.w;
    }
    return 1.f;
}

template <int MB>
__global__ void __launch_bounds__(kTcWarps * 32, 1) gemm_tc_kernel(const TcArgs args) {
    using C = TcCfg<MB>;
    extern __shared__ __align__(1024) uint8_t tsm[];
    const Prob &a = args.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cr = (a.cl > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int D = args.depth;
    // shared memory: [x images kTcSets x 2][ring kTcComputeWarps x D][scales
    // kTcComputeWarps x P x 32][red 128 x MB][bars][tmem slot, abort]
    uint8_t *ximg = tsm;
    uint8_t *ring_base = ximg + (size_t)kTcSets * 2 * C::XBYTES;
    float *sbuf = reinterpret_cast<float *>(ring_base + (size_t)kTcComputeWarps * D * kStageBytes);
    float *red = sbuf + kTcComputeWarps * C::P * 32;
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + 128 * MB);
    uint64_t *full = bars + kTcComputeWarps * D;  // [kTcSets][P]
    uint64_t *done = full + kTcSets * C::P;        // [kTcSets][P]
    uint64_t *fin = done + kTcSets * C::P;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    // this CTA's share of the units of every block it visits
    const int OB = a.U - a.S;
    const int sg0 = split_at(a.S, cr, a.cl), ob0 = split_at(OB, cr, a.cl);
    const int nsg = split_at(a.S, cr + 1, a.cl) - sg0;
    const int nunits = nsg + (split_at(OB, cr + 1, a.cl) - ob0);
    const int bstride = (int)(gridDim.x / a.cl);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTcTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int b = 0; b < kTcSets * C::P; ++b) {
            mbar_init(smem_u32(&full[b]), 128u);
            mbar_init(smem_u32(&done[b]), 1u);
        }
        mbar_init(smem_u32(fin), 1u);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    Ring ring;
    if (warp < kTcComputeWarps)
        ring_init(ring, ring_base + (size_t)warp * D * kStageBytes, bars + warp * D, D, lane);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    if (warp < kTcComputeWarps) {
        // ------------------------------------------------ compute warps
        const int j = warp >> 2, r = warp & 3, tid = threadIdx.x - 128 * j;
        const uint32_t tl = tmem + ((uint32_t)(32 * r) << 16);
        uint64_t *fullj = full + j * C::P, *donej = done + j * C::P;
        float *sb = sbuf + (warp * C::P) * 32 + lane;
        // issue iterator (ring) and x iterator run ahead of the work iterator
        int iblk = blockIdx.x / a.cl, ilu = j;
        auto advance = [&](int &blk, int &lu) {
            lu += kTcSets;
            if (lu >= nunits) {
                blk += bstride;
                lu = j;
            }
        };
        if (j >= nunits) iblk = args.nblk;  // this set has no units
        for (int d = 0; d < D && iblk < args.nblk; ++d) {
            const int t = 4 * iblk + r;
            if (t < a.T) ring_issue(ring, a, t, tc_unit(a, sg0, nsg, ob0, ilu), lane);
            else ring.issued += ring.ok ? 1 : 0;  // keeps issue and acquire counts aligned
            advance(iblk, ilu);
        }
        pdl_wait();
        int xblk = blockIdx.x / a.cl, xlu = j;
        if (j >= nunits) xblk = args.nblk;
        TcX<MB> xp;
        if (xblk < args.nblk) tc_load_x<MB>(a, tc_unit(a, sg0, nsg, ob0, xlu), tid, xp);
        advance(xblk, xlu);

        int gi = 0, gc = 0, xl = 0;
        int lastg[2] = {-1, -1};
        float y[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) y[m] = 0.f;
        auto consume = [&]() {
            const int b = gc % C::P;
            if (lane == 0) tc_wait(smem_u32(&donej[b]), (uint32_t)(gc / C::P) & 1u, abort);
            __syncwarp();
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            float dv[MB];
            tmem_ld_d<MB>(tl + (uint32_t)(C::DCOL + (j * C::P + b) * MB), dv);
            const float s = sb[b * 32];
            const float2 s2 = make_float2(s, s);
#pragma unroll
            for (int m = 0; m < MB; m += 2) {
                const float2 r2 = __ffma2_rn(s2, make_float2(dv[m], dv[m + 1]), make_float2(y[m], y[m + 1]));
                y[m] = r2.x;
                y[m + 1] = r2.y;
            }
            ++gc;
        };

        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride) {
            const int t = 4 * blk + r;
            const bool active = t < a.T;
            for (int lu = j; lu < nunits; lu += kTcSets, ++xl) {
                const int u = tc_unit(a, sg0, nsg, ob0, lu);
                uint8_t *xb = ximg + (size_t)(j * 2 + (xl & 1)) * C::XBYTES;
                // the MMAs of unit xl - 2 read this x buffer: wait for them
                while (gc <= lastg[xl & 1]) consume();
                tc_store_x<MB>(a, u, tid, xp, xb);
                if (xblk < args.nblk) {
                    tc_load_x<MB>(a, tc_unit(a, sg0, nsg, ob0, xlu), tid, xp);
                    advance(xblk, xlu);
                }
                const uint8_t *stage = nullptr;
                if (active) stage = ring_acquire(ring, lane);
                else if (ring.ok) ++ring.consumed;
                __syncwarp();
                const int ngr = tc_groups(a, u);
                for (int g = 0; g < ngr; ++g) {
                    const int b = gi % C::P;
                    uint32_t av[16];
                    const float s = tc_build_a(a, u, g, stage, lane, av);
                    tmem_st16(tl + (uint32_t)((j * C::P + b) * 16), av);
                    sb[b * 32] = s;
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    mbar_arrive(smem_u32(&fullj[b]));
                    ++gi;
                    if (gi - gc > C::L) consume();
                }
                lastg[xl & 1] = gi - 1;
                if (active) ring_release(ring);
                if (iblk < args.nblk) {
                    const int ti = 4 * iblk + r;
                    if (ti < a.T) ring_issue(ring, a, ti, tc_unit(a, sg0, nsg, ob0, ilu), lane);
                    else ring.issued += ring.ok ? 1 : 0;
                    advance(iblk, ilu);
                }
            }
            while (gc < gi) consume();
            // block end: set 1 hands its sums to set 0, which stores the rows
            // (or, in a cluster, leaves them for the rank-ordered reduction)
            if (j == 1) {
#pragma unroll
                for (int m = 0; m < MB; ++m) red[(32 * r + lane) * MB + m] = y[m];
            }
            named_sync(1, 32 * kTcComputeWarps);
            if (j == 0) {
#pragma unroll
                for (int m = 0; m < MB; ++m) y[m] += red[(32 * r + lane) * MB + m];
                if (a.cl > 1) {
#pragma unroll
                    for (int m = 0; m < MB; ++m) red[(32 * r + lane) * MB + m] = y[m];
                } else if (active) {
#pragma unroll
                    for (int m = 0; m < MB; ++m) store_y(a, t, lane, m, y[m]);
                }
            }
            named_sync(1, 32 * kTcComputeWarps);
#pragma unroll
            for (int m = 0; m < MB; ++m) y[m] = 0.f;
        }
        ring_drain(ring);
    } else if (lane == 0) {
        // ------------------------------------------------ MMA issuer (one lane)
        pdl_wait();
        const uint32_t idesc = bf16_idesc<MB>();
        int gis[kTcSets] = {}, xls[kTcSets] = {};
        bool any = false;
        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride) {
            for (int lub = 0; lub < nunits; lub += kTcSets) {
                int ngr[kTcSets], gmax = 0;
#pragma unroll
                for (int s = 0; s < kTcSets; ++s) {
                    ngr[s] = lub + s < nunits ? tc_groups(a, tc_unit(a, sg0, nsg, ob0, lub + s)) : 0;
                    gmax = max(gmax, ngr[s]);
                }
                for (int g = 0; g < gmax; ++g) {
#pragma unroll
                    for (int s = 0; s < kTcSets; ++s) {
                        if (g >= ngr[s]) continue;
                        const int b = gis[s] % C::P;
                        const bool ok = tc_wait(smem_u32(&full[s * C::P + b]), (uint32_t)(gis[s] / C::P) & 1u, abort);
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        if (ok) {
                            const uint32_t xs = smem_u32(ximg + (size_t)(s * 2 + (xls[s] & 1)) * C::XBYTES) +
                                                (uint32_t)(2 * g * C::KSTEP);
                            const uint32_t ta = tmem + (uint32_t)((s * C::P + b) * 16);
                            const uint32_t td = tmem + (uint32_t)(C::DCOL + (s * C::P + b) * MB);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint64_t bdesc = umma_desc(xs + (uint32_t)(h * C::KSTEP), 128u, 256u);
                                asm volatile(
                                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
                                    "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(td),
                                    "r"(ta + 8u * h), "l"(bdesc), "r"((uint32_t)h), "r"(idesc)
                                    : "memory");
                            }
                            any = true;
                        }
                        asm volatile(
                            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                smem_u32(&done[s * C::P + b]))
                            : "memory");
                        ++gis[s];
                    }
                }
#pragma unroll
                for (int s = 0; s < kTcSets; ++s)
                    if (lub + s < nunits) ++xls[s];
            }
        }
        // every MMA of this CTA has completed before TMEM is released
        if (any) {
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    smem_u32(fin))
                : "memory");
            tc_wait(smem_u32(fin), 0u, abort);
        }
    }
    __syncwarp();

    // cluster split (one block per cluster): rank 0 adds the ranks' sums in rank order
    if (a.cl > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int blk = blockIdx.x / a.cl;
        if (cr == 0 && warp < 4) {
            const int t = 4 * blk + warp;
            float yv[MB];
#pragma unroll
            for (int m = 0; m < MB; ++m) yv[m] = 0.f;
            for (int rk = 0; rk < a.cl; ++rk) {
                const float *rp = cluster.map_shared_rank(red, rk) + (32 * warp + lane) * MB;
#pragma unroll
                for (int m = 0; m < MB; ++m) yv[m] += rp[m];
            }
            if (t < a.T) {
#pragma unroll
                for (int m = 0; m < MB; ++m) store_y(a, t, lane, m, yv[m]);
            }
        }
        cluster.sync();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTcTmemCols));
    }
}

size_t tc_smem_bytes(int MB, int depth) {
    const int P = MB == 32 ? TcCfg<32>::P : TcCfg<16>::P;
    return (size_t)kTcSets * 2 * 256 * MB * 2 + (size_t)kTcComputeWarps * depth * kStageBytes +
           (size_t)kTcComputeWarps * P * 32 * 4 + (size_t)128 * MB * 4 +
           (size_t)(kTcComputeWarps * depth + 2 * kTcSets * P + 1) * 8 + 16;
}

template <int MB>
spectra_status run_tc(const Prob &a0, const DeviceInfo &dev, cudaStream_t s) {
    static bool done[64];
    TcArgs args;
    args.p = a0;
    const Geometry g = Geometry::of(a0.n, a0.k, a0.n_o);
    const int64_t nblk = cdiv(g.T, 4);
    const int units = units_of(g);
    int cl = 1;
    int64_t grid = nblk;
    if (nblk >= dev.sm_count) {
        grid = dev.sm_count;  // persistent over the blocks
    } else {
        // one block per cluster, the clusters filling the SMs once
        cl = (int)(dev.sm_count / nblk);
        if (cl > 8) cl = 8;
        if (cl > units) cl = units;
        if (cl < 1) cl = 1;
        grid = nblk * cl;
    }
    args.p.cl = cl;
    args.nblk = (int)nblk;
    int depth = 4;
    while (depth > 1 && tc_smem_bytes(MB, depth) > dev.smem_optin) --depth;
    args.depth = depth;
    const size_t smem = tc_smem_bytes(MB, depth);
    if (smem > dev.smem_optin) return SPECTRA_ERR_SHAPE;
    cudaError_t e = prepare_kernel(gemm_tc_kernel<MB>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    e = launch_kernel(gemm_tc_kernel<MB>, args, (unsigned)grid, smem, kTcWarps, cl, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

}  // namespace

spectra_status device_error(bool *raised, cudaStream_t s) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    *raised = v != 0;
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
    const Geometry g = Geometry::of(l.n, l.k, l.n_outliers);
    if (m >= 16) {
        // a real dense contraction: the tensor-core path
        Prob a;
        fill_prob(a, l, g, x, m, y, ytype);
        return m <= 16 ? run_tc<16>(a, dev, s) : run_tc<32>(a, dev, s);
    }
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
        const Geometry g = Geometry::of(layers[i].n, layers[i].k, layers[i].n_outliers);
        fill_prob(args.probs[i], layers[i], g, xs[i], 1, ys[i], ytype);
    }
    return run_persistent<1>(args, count, dev, s);
}

}  // namespace spectra
