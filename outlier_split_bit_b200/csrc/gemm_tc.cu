// gemm_tc.cu -- y = x W_hat^T for 8 <= m <= 32 batch rows on the fifth-
// generation tensor cores (tcgen05, sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: the Group-32 4-bit
// weights are dequantised in registers and the BF16 outlier channels enter
// the same product.  For a batch of 8 or more rows the product is a real
// dense contraction, so the decoded operand goes to the tensor cores (8..16
// rows run the 16-row variant; its surplus rows are computed and dropped).
#include <atomic>

#include "stream.cuh"

namespace spectra {
namespace {

// ---------------------------------------------------------------- design
//
// A CTA owns blocks of 128 rows (4 tiles; TMEM lane = row) and streams their
// units (super-groups of 8 groups, outlier batches of up to 8 octets) with:
//
//  * SETS sets of four compute warps.  Set j takes every SETS-th unit of the
//    block; warp 4j + r owns tile r (rows 32r..32r+31) and keeps its own
//    cp.async.bulk ring of that tile's units.  Per group of 32 columns each
//    lane writes its row of the A operand into TMEM: the dequantised weights
//    s * (c - z) rounded once to FP16 (c - z is exact in FP16, then one
//    round-to-nearest-even multiply by the FP16 scale).  Outlier columns enter
//    with their exact BF16 weights.  The set's threads also stage x as the B
//    operand: FP16 for the bulk (BF16 x converted, exact in FP16's normal
//    range), BF16 for the outlier columns.
//  * one MMA warp per set, whose elected lane issues the set's tcgen05.mma
//    (kind::f16, M = 128, N = MB, K = 16; A from TMEM, B from shared memory)
//    into the set's FP32 accumulator for the block in TMEM, so the scales
//    need no FP32 epilogue per group: the row sums stay in the tensor core
//    until the block ends.  The sets' accumulators are independent MMA
//    dependency chains (so the tensor pipe overlaps them, and no issuer waits
//    for another set), and a set's consecutive MMAs may rotate over NCH
//    accumulators; all are summed in a fixed order when the block is read.
//
// Groups travel in chunks of H: the warps of a set store H groups' A operands
// into one of the set's Q = 2 TMEM slots and arrive once on full[slot]; the
// MMA lane waits, issues 2H MMAs and commits to done[slot].  A slot (and the
// x image of the unit two units back) is rewritten only after done[] of the
// chunk that last used it, so the MMAs that read them have completed.  At a
// block end each MMA lane commits to its set's dready[block & 1]; set 0 reads
// every set's accumulator back (deferred until it has built the next block's
// first chunk, so the MMA pipe stays fed) and arrives on the sets'
// dfree[block & 1], which each MMA lane awaits before the block two later
// overwrites its accumulator.
//
// Accuracy: each weight carries one FP16 rounding (relative 2^-11) and FP32
// accumulation, well inside |y - y_ref| <= 2e-3 * sum|w_hat x| + 1e-5; with x
// a unit vector e_j, y is column j of W_hat rounded to FP16 (exactly), plus
// the column's BF16 weight when j is an outlier.  Range: an FP16 operand that
// overflows (|x| > 65504 in a bulk column, or a group scale of 4368 or more)
// makes the row's sum non-finite; the read-back raises the RANGE flag of
// spectra_device_status for any non-finite output.  Every wait is bounded by
// a one-second %globaltimer limit and sleeps on the mbarrier's suspend hint.
constexpr int kTcTmemCols = 512;

template <int MB_, int SETS_, int H_, int NCH_>
struct TcCfg {
    static constexpr int MB = MB_;
    static constexpr int SETS = SETS_;             // warp sets
    static constexpr int H = H_;                   // groups per handshake (a chunk)
    static constexpr int Q = 2;                    // chunk slots per set
    static constexpr int NCH = NCH_;               // accumulator chains per block
    static constexpr int CW = 4 * SETS;            // compute warps
    static constexpr int WARPS = CW + SETS;        // + one MMA warp per set
    static constexpr int ACOLS = H * 16;           // TMEM columns of one chunk's A operands
    static constexpr int DCOL = SETS * Q * ACOLS;  // A slots below, accumulators from here
    static constexpr int XBYTES = 256 * MB * 2;    // x image of one unit (256 columns)
    static constexpr int KSTEP = MB * 32;          // bytes of one 16-column K step of x
    static_assert(DCOL % 32 == 0, "accumulator alignment");
    static_assert(DCOL + SETS * 2 * NCH * MB <= kTcTmemCols, "TMEM budget");
    static_assert(H >= 1 && H <= 8 && NCH >= 1 && NCH <= 4, "chunk shape");
};

// 16 rows: three sets, one accumulator each; 32 rows: two sets, two
// accumulators each.  Chunks of four groups.
using TcCfg16 = TcCfg<16, 3, 4, 1>;
using TcCfg32 = TcCfg<32, 2, 4, 2>;

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

// Instruction descriptor of kind::f16: D = F32 (bits 4-5 = 1), A and B of the
// same type (format at bits 7 and 10: 0 = F16, 1 = BF16), both K-major,
// N = MB (>> 3 at bit 17), M = 128 (>> 4 at bit 24).
template <int MB>
__device__ __forceinline__ uint32_t f16_idesc(bool bf16) {
    const uint32_t t = bf16 ? 1u : 0u;
    return (1u << 4) | (t << 7) | (t << 10) | ((uint32_t)(MB >> 3) << 17) | (8u << 24);
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

// A bounded mbarrier wait that also turns every later wait of the CTA into a
// no-op once one has timed out (`abort` is CTA-shared).
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kWaitRounds; ++i) {
        if (mbar_try(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > kWaitNs) break;
    }
    *abort = 1;
    atomicOr(&g_device_error, 1u);
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
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
        // products land in accumulator columns, or K steps, that are never used)
        const int nw = 4 * min(8, a.G - 8 * u);
#pragma unroll
        for (int i = 0; i < MB / 4; ++i) {
            const int c = tid + 128 * i, m = min(c % MB, a.m - 1), W = min(c / MB, nw - 1);
            xp.v[i] = a.bidx == nullptr
                          ? __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)m * a.kx + 256 * u + 8 * W))
                          : bulk_x8_gather(a, m, 256 * u + 8 * W);
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
            const uint16_t *row = a.x + (size_t)min(m, a.m - 1) * a.kx;
            uint32_t h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = (uint32_t)__ldg(row + max(ix[e], 0));
            xp.v[i] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                 h[6] | (h[7] << 16));
        }
    }
}

// FP16 pair (lo, hi) of two BF16 values given in the high halves of 32-bit
// words (each exact as FP32; one rounding to FP16).
__device__ __forceinline__ uint32_t f16_pair(uint32_t lo_bits, uint32_t hi_bits) {
    const __half2 h = __floats2half2_rn(__uint_as_float(lo_bits), __uint_as_float(hi_bits));
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Write the prefetched x of unit u as the B image: chunk W goes to K step
// W / 2, core-matrix column W % 2.  Super-group chunks become FP16 pairs in
// the decoder's order (x0, x4), (x1, x5), (x2, x6), (x3, x7); outlier chunks
// stay BF16 in slot order.
template <int MB>
__device__ __forceinline__ void tc_store_x(const Prob &a, int u, int tid, const TcX<MB> &xp,
                                           uint8_t *xb) {
    if (u < a.S) {
#pragma unroll
        for (int i = 0; i < MB / 4; ++i) {
            const int c = tid + 128 * i, m = c % MB, W = c / MB;
            const uint4 v = xp.v[i];  // (x0, x1), (x2, x3), (x4, x5), (x6, x7)
            const uint4 p = make_uint4(f16_pair(v.x << 16, v.z << 16),
                                       f16_pair(v.x & 0xFFFF0000u, v.z & 0xFFFF0000u),
                                       f16_pair(v.y << 16, v.w << 16),
                                       f16_pair(v.y & 0xFFFF0000u, v.w & 0xFFFF0000u));
            *reinterpret_cast<uint4 *>(xb + (W >> 1) * (MB * 32) + (m >> 3) * 256 +
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
            *reinterpret_cast<uint4 *>(xb + (o >> 1) * (MB * 32) + (m >> 3) * 256 +
                                       (o & 1) * 128 + (m & 7) * 16) =
                make_uint4(v.x & k0, v.y & k1, v.z & k2, v.w & k3);
        }
    }
}

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Shared-memory loads by 32-bit address (the ring stages are shared memory).
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// MB consecutive FP32 accumulator columns of this warp's 32 lanes.
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

// The A operand of bulk group g for one row (lane): 16 TMEM columns of FP16
// pairs s * (c - z), column 4w + s holding the codes of columns 8w + s (low)
// and 8w + s + 4 (high) of the group.  1024 + c is exact in FP16 (10
// mantissa bits), so the subtraction of 1024 + z is exact and the multiply
// by the scale is the one rounding.
__device__ __forceinline__ void tc_build_a_bulk(uint32_t sa, int g, int lane, uint32_t *av) {
    const uint4 q = lds128(sa + g * 512 + lane * 16);
    const uint32_t sw = lds32(sa + 4096 + lane * 16 + (g >> 1) * 4);
    const uint32_t zw = lds32(sa + 4608 + lane * 4);
    const uint32_t ss = __byte_perm(sw, 0u, (g & 1) ? 0x3232u : 0x1010u);    // (s, s)
    const uint32_t zz = (0x6400u | ((zw >> (4 * g)) & 0xFu)) * 0x00010001u;  // (1024 + z, 1024 + z)
    const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint32_t p = ((wv[w] >> (4 * s)) & 0x000F000Fu) | 0x64006400u;  // (1024 + c, 1024 + c')
            av[4 * w + s] = f16x2_mul(f16x2_sub(p, zz), ss);
        }
    }
}

// The A operand of outlier group g (octets 4g..4g+3) of batch unit u: the
// exact BF16 weights, zero past the batch's last octet.
__device__ __forceinline__ void tc_build_a_outlier(const Prob &a, int u, int g, uint32_t sa, int lane,
                                                   uint32_t *av) {
    const int nv = min(kOB, a.O8 - kOB * (u - a.S));
#pragma unroll
    for (int o = 0; o < 4; ++o) {
        uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
        if (4 * g + o < nv) w4 = lds128(sa + (4 * g + o) * 512 + lane * 16);
        av[4 * o + 0] = w4.x;
        av[4 * o + 1] = w4.y;
        av[4 * o + 2] = w4.z;
        av[4 * o + 3] = w4.w;
    }
}

template <typename C>
__global__ void __launch_bounds__(C::WARPS * 32, 1) gemm_tc_kernel(const TcArgs args) {
    constexpr int MB = C::MB;
    extern __shared__ __align__(1024) uint8_t tsm[];
    const Prob &a = args.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cr = (a.cl > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int D = args.depth;
    // shared memory: [x images SETS x 2][ring CW x D][bars][tmem slot, abort].
    // In a cluster (one block per CTA) set 0's x images hold the block's
    // 128 x MB partial sums at the end, once every MMA has completed.
    uint8_t *ximg = tsm;
    uint8_t *ring_base = ximg + (size_t)C::SETS * 2 * C::XBYTES;
    float *red = reinterpret_cast<float *>(ximg);
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring_base + (size_t)C::CW * D * kStageBytes);
    uint64_t *full = bars + C::CW * D;        // [SETS][Q]
    uint64_t *done = full + C::SETS * C::Q;   // [SETS][Q]
    uint64_t *dready = done + C::SETS * C::Q; // [SETS][2]
    uint64_t *dfree = dready + C::SETS * 2;   // [SETS][2]
    uint64_t *fin = dfree + C::SETS * 2;      // [SETS]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + C::SETS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    // this CTA's share of the units of every block it visits: a contiguous
    // range of the block's unit list (super-groups, then outlier batches),
    // the same number of units per rank (with cl <= U every rank has at
    // least one).  Units are counted, not weighted by their groups: a
    // super-group of eight groups and an outlier batch of two measured about
    // the same cost per unit (the batch's gathered x is a chain of two
    // dependent loads per column, behind a single chunk)
    const int u0 = split_at(a.U, cr, a.cl), u1 = split_at(a.U, cr + 1, a.cl);
    const int sg0 = u0, nsg = max(0, min(u1, a.S) - u0);
    const int ob0 = max(u0, a.S) - a.S;
    const int nunits = u1 - u0;
    const int bstride = (int)(gridDim.x / a.cl);
    // MMAs of one block per set (the same for every block this CTA visits):
    // two per group
    int nmma[C::SETS];
#pragma unroll
    for (int j = 0; j < C::SETS; ++j) {
        nmma[j] = 0;
        for (int lu = j; lu < nunits; lu += C::SETS) nmma[j] += 2 * tc_groups(a, tc_unit(a, sg0, nsg, ob0, lu));
    }

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTcTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 32) {
        for (int b = 0; b < C::SETS * C::Q; ++b) {
            mbar_init(smem_u32(&full[b]), 4u);  // one arrival per compute warp of the set
            mbar_init(smem_u32(&done[b]), 1u);
        }
        for (int b = 0; b < C::SETS * 2; ++b) {
            mbar_init(smem_u32(&dready[b]), 1u);
            mbar_init(smem_u32(&dfree[b]), 4u);  // one arrival per warp of set 0
        }
        for (int j = 0; j < C::SETS; ++j) mbar_init(smem_u32(&fin[j]), 1u);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    Ring ring;
    if (warp < C::CW)
        ring_init(ring, ring_base + (size_t)warp * D * kStageBytes, bars + warp * D, D, lane);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    if (warp < C::CW) {
        // ------------------------------------------------ compute warps
        const int j = warp >> 2, r = warp & 3, tid = threadIdx.x - 128 * j;
        const uint32_t tl = tmem + ((uint32_t)(32 * r) << 16);
        uint64_t *fullj = full + j * C::Q, *donej = done + j * C::Q;
        // issue iterator (ring) and x iterator run ahead of the work iterator
        int iblk = blockIdx.x / a.cl, ilu = j;
        auto advance = [&](int &blk, int &lu) {
            lu += C::SETS;
            if (lu >= nunits) {
                blk += bstride;
                lu = j;
            }
        };
        if (j >= nunits) iblk = args.nblk;  // this set has no units
        for (int d = 0; d < D && iblk < args.nblk; ++d) {
            const int t = 4 * iblk + r;
            if (t < a.T) ring_issue(ring, a, t, tc_unit(a, sg0, nsg, ob0, ilu), lane);
            else ring_advance_issue(ring);  // keeps issue and acquire counts aligned
            advance(iblk, ilu);
        }
        pdl_wait();
        int xblk = blockIdx.x / a.cl, xlu = j;
        if (j >= nunits) xblk = args.nblk;
        TcX<MB> xp;
        if (xblk < args.nblk) tc_load_x<MB>(a, tc_unit(a, sg0, nsg, ob0, xlu), tid, xp);
        advance(xblk, xlu);

        // Set 0 reads each block's accumulator back and stores its rows (or,
        // in a cluster, leaves them for the rank-ordered reduction).
        auto read_back = [&](int b, int blk) {
            float acc[MB];
#pragma unroll
            for (int m = 0; m < MB; ++m) acc[m] = 0.f;
#pragma unroll
            for (int js = 0; js < C::SETS; ++js) {
                tc_wait(smem_u32(&dready[js * 2 + (b & 1)]), (uint32_t)(b >> 1) & 1u, abort);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t td = tl + (uint32_t)(C::DCOL + ((js * 2 + (b & 1)) * C::NCH) * MB);
#pragma unroll
                for (int c = 0; c < C::NCH; ++c) {
                    if (c < nmma[js]) {  // CTA-uniform: this accumulator was written in the block
                        float t2[MB];
                        tmem_ld_d<MB>(td + (uint32_t)(c * MB), t2);
#pragma unroll
                        for (int m = 0; m < MB; ++m) acc[m] += t2[m];
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int js = 0; js < C::SETS; ++js) mbar_arrive(smem_u32(&dfree[js * 2 + (b & 1)]));
            }
            const int t = 4 * blk + r;
            if (a.cl > 1) {
#pragma unroll
                for (int m = 0; m < MB; ++m) red[m * 128 + 32 * r + lane] = acc[m];
            } else if (t < a.T) {
                bool bad = false;
#pragma unroll
                for (int m = 0; m < MB; ++m) {
                    store_y(a, t, lane, m, acc[m]);
                    bad |= (m < a.m) && !isfinite(acc[m]);
                }
                if (bad && 32 * t + lane < a.n) atomicOr(&g_device_error, 2u);
            }
        };

        int c = 0, xl = 0, b = 0;     // chunks, units and blocks of this set so far
        int pend = -1, pend_blk = 0;  // set 0: a block whose accumulator is still to be read
        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride, ++b) {
            const int t = 4 * blk + r;
            const bool active = t < a.T;
            for (int lu = j; lu < nunits; lu += C::SETS, ++xl) {
                const int u = tc_unit(a, sg0, nsg, ob0, lu);
                const bool bulk = u < a.S;
                uint8_t *xb = ximg + (size_t)(j * 2 + (xl & 1)) * C::XBYTES;
                const uint8_t *stage = nullptr;
                if (active) stage = ring_acquire(ring, lane);
                else ring_advance_consume(ring);
                __syncwarp();
                const uint32_t sa = stage ? smem_u32(stage) : 0u;
                const int ngr = tc_groups(a, u);
                for (int g0 = 0; g0 < ngr; g0 += C::H, ++c) {
                    const int q = c & 1;
                    // the slot's previous chunk (and, at a unit's start, every
                    // MMA that read this x image two units back) has completed
                    if (c >= C::Q) tc_wait(smem_u32(&donej[q]), (uint32_t)((c - C::Q) >> 1) & 1u, abort);
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (g0 == 0) {
                        tc_store_x<MB>(a, u, tid, xp, xb);
                        if (xblk < args.nblk) {
                            tc_load_x<MB>(a, tc_unit(a, sg0, nsg, ob0, xlu), tid, xp);
                            advance(xblk, xlu);
                        }
                    }
                    const int nh = min(C::H, ngr - g0);
#pragma unroll
                    for (int h = 0; h < C::H; ++h) {
                        if (h < nh) {  // warp-uniform
                            uint32_t av[16];
                            if (!stage) {
#pragma unroll
                                for (int i = 0; i < 16; ++i) av[i] = 0u;
                            } else if (bulk) {
                                tc_build_a_bulk(sa, g0 + h, lane, av);
                            } else {
                                tc_build_a_outlier(a, u, g0 + h, sa, lane, av);
                            }
                            tmem_st16(tl + (uint32_t)((j * C::Q + q) * C::ACOLS + h * 16), av);
                        }
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&fullj[q]));
                    if (pend >= 0) {  // set 0 only: the previous block, now that this one is fed
                        read_back(pend, pend_blk);
                        pend = -1;
                    }
                }
                if (active) ring_release(ring);
                if (iblk < args.nblk) {
                    const int ti = 4 * iblk + r;
                    if (ti < a.T) ring_issue(ring, a, ti, tc_unit(a, sg0, nsg, ob0, ilu), lane);
                    else ring_advance_issue(ring);
                    advance(iblk, ilu);
                }
            }
            if (j == 0) {
                pend = b;
                pend_blk = blk;
            }
        }
        if (pend >= 0) read_back(pend, pend_blk);
        ring_drain(ring);
    } else if (lane == 0) {
        // ------------------------------------------------ MMA issuer of set j (one lane)
        const int j = warp - C::CW;
        int cj = 0, xj = 0, b = 0;  // chunks, units and blocks of this set so far
        const uint32_t x0 = smem_u32(ximg + (size_t)(j * 2) * C::XBYTES);
        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride, ++b) {
            // this set's accumulator two blocks back has been read
            if (b >= 2) tc_wait(smem_u32(&dfree[j * 2 + (b & 1)]), (uint32_t)((b - 2) >> 1) & 1u, abort);
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t td0 = tmem + (uint32_t)(C::DCOL + ((j * 2 + (b & 1)) * C::NCH) * MB);
            int mi = 0;  // this set's MMAs of the block so far
            for (int lu = j; lu < nunits; lu += C::SETS, ++xj) {
                const int u = tc_unit(a, sg0, nsg, ob0, lu);
                const int ngr = tc_groups(a, u);
                const uint32_t idesc = f16_idesc<MB>(u >= a.S);
                const uint32_t xs0 = x0 + (uint32_t)((xj & 1) * C::XBYTES);
                for (int g0 = 0; g0 < ngr; g0 += C::H, ++cj) {
                    const int q = cj & 1;
                    const int nh = min(C::H, ngr - g0);
                    const bool ok = tc_wait(smem_u32(&full[j * C::Q + q]), (uint32_t)(cj >> 1) & 1u, abort);
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (ok) {
                        const uint32_t ta0 = tmem + (uint32_t)((j * C::Q + q) * C::ACOLS);
                        for (int h = 0; h < nh; ++h) {
#pragma unroll
                            for (int k = 0; k < 2; ++k) {
                                const uint32_t xs = xs0 + (uint32_t)((2 * (g0 + h) + k) * C::KSTEP);
                                const uint64_t bdesc = umma_desc(xs, 128u, 256u);
                                const uint32_t td = td0 + (uint32_t)((mi % C::NCH) * MB);
                                // the first product into an accumulator in this block overwrites it
                                const uint32_t accum = mi >= C::NCH ? 1u : 0u;
                                ++mi;
                                asm volatile(
                                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
                                    "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(td),
                                    "r"(ta0 + (uint32_t)(h * 16 + 8 * k)), "l"(bdesc), "r"(accum), "r"(idesc)
                                    : "memory");
                            }
                        }
                    }
                    // one commit per chunk: done[] fires when all its MMAs completed
                    mma_commit(smem_u32(&done[j * C::Q + q]));
                }
            }
            // the set's accumulator is complete once every MMA so far has completed
            mma_commit(smem_u32(&dready[j * 2 + (b & 1)]));
        }
        // every MMA this lane issued has completed before TMEM is released
        mma_commit(smem_u32(&fin[j]));
        tc_wait(smem_u32(&fin[j]), 0u, abort);
    }
    __syncwarp();

    // cluster split (one block per cluster): rank cr adds the ranks' sums of
    // batch rows m = cr, cr + cl, ... in rank order and stores them
    if (a.cl > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int blk = blockIdx.x / a.cl;
        const int t = 4 * blk + warp;
        if (warp < 4 && t < a.T) {
            const float *rp[8];
#pragma unroll
            for (int rk = 0; rk < 8; ++rk)
                rp[rk] = cluster.map_shared_rank(red, rk < a.cl ? rk : 0) + 32 * warp + lane;
            bool bad = false;
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                if (m % a.cl != cr || m >= a.m) continue;  // CTA-uniform
                float v[8];
#pragma unroll
                for (int rk = 0; rk < 8; ++rk) v[rk] = rp[rk][m * 128];
                float yv = 0.f;
#pragma unroll
                for (int rk = 0; rk < 8; ++rk)
                    if (rk < a.cl) yv += v[rk];
                store_y(a, t, lane, m, yv);
                bad |= !isfinite(yv);
            }
            if (bad && 32 * t + lane < a.n) atomicOr(&g_device_error, 2u);
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

template <typename C>
size_t tc_smem_bytes(int depth) {
    return (size_t)C::SETS * 2 * C::XBYTES + (size_t)C::CW * depth * kStageBytes +
           (size_t)(C::CW * depth + 2 * C::SETS * C::Q + 5 * C::SETS) * 8 + 16;
}

// Clusters of `cl` CTAs of gemm_tc_kernel<C> (with `smem` bytes each) the
// device holds at once; cached per device and cluster size, 0 if unknown.
template <typename C>
int tc_max_clusters(int cl, size_t smem, const DeviceInfo &dev) {
    static std::atomic<int> cache[64][9];
    if (dev.device < 0 || dev.device >= 64 || cl < 1 || cl > 8) return 0;
    int v = cache[dev.device][cl].load(std::memory_order_relaxed);
    if (v > 0) return v - 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(cl * dev.sm_count), 1, 1);
    cfg.blockDim = dim3(C::WARPS * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cl;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<C>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cache[dev.device][cl].store(n + 1, std::memory_order_relaxed);
    return n;
}

template <typename C>
spectra_status run_tc(const Prob &a0, const DeviceInfo &dev, cudaStream_t s) {
    static bool done[64];
    TcArgs args;
    args.p = a0;
    const Geometry g = Geometry::of(a0.n, a0.k, a0.n_o);
    const int64_t nblk = cdiv(g.T, 4);
    const int units = units_of(g);
    int depth = 2;  // two units in flight per warp
    while (depth > 1 && tc_smem_bytes<C>(depth) > dev.smem_optin) --depth;
    const size_t smem = tc_smem_bytes<C>(depth);
    if (smem > dev.smem_optin) return SPECTRA_ERR_SHAPE;
    cudaError_t e = prepare_kernel(gemm_tc_kernel<C>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
    int cl = 1;
    int64_t grid = nblk;
    if (nblk >= dev.sm_count) {
        grid = dev.sm_count;  // persistent over the blocks
    } else {
        // one block per cluster: the largest cluster size whose nblk
        // clusters the device holds at once (a cluster lives inside one GPC,
        // so sizes that do not divide a GPC's SMs leave some idle and would
        // push clusters into a second wave)
        cl = (int)(dev.sm_count / nblk);
        if (cl > 8) cl = 8;
        if (cl > units) cl = units;
        while (cl > 1 && tc_max_clusters<C>(cl, smem, dev) < nblk) --cl;
        if (cl < 1) cl = 1;
        grid = nblk * cl;
    }
    args.p.cl = cl;
    args.nblk = (int)nblk;
    args.depth = depth;
    e = launch_kernel(gemm_tc_kernel<C>, args, (unsigned)grid, smem, C::WARPS, cl, s);
    return e == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
}

}  // namespace

spectra_status launch_tc(const spectra_layer &l, const uint16_t *x, int m, void *y, int ytype,
                         cudaStream_t s, const DeviceInfo &dev) {
    const Geometry g = Geometry::of(l.n, bulk_cols(l), l.n_outliers);
    Prob a;
    fill_prob(a, l, g, x, m, y, ytype);
    return m <= 16 ? run_tc<TcCfg16>(a, dev, s) : run_tc<TcCfg32>(a, dev, s);
}

spectra_status tc_device_error(unsigned int *bits, cudaStream_t s) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    *bits = v;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                    s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
    }
    return SPECTRA_OK;
}

}  // namespace spectra
