// gemm_tc.cu -- y = x W_hat^T for 8 <= m <= 32 batch rows on the fifth-
// generation tensor cores (tcgen05, sm_100a).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: the Group-32 4-bit
// weights are dequantised in registers and the BF16 outlier channels enter
// the same product.  For a batch of 8 or more rows the product is a real
// dense contraction, so the decoded operand goes to the tensor cores (8..16
// rows run the 16-row variant; its surplus rows are computed and dropped).
#include "stream.cuh"

namespace spectra {
namespace {

// ---------------------------------------------------------------- tensor-core path (M = 16..32)
//
// y[m][n] for 8 <= m_rows <= 32 (MB = 16 or 32 batch rows) on the fifth-
// generation tensor cores.  A CTA owns blocks of 128 rows (4 tiles; TMEM
// lane = row) and streams their units (super-groups, outlier batches) with
// two kinds of warps:
//
//  * SETS sets of four compute warps (three at 16 rows, two at 32).  Set j
//    takes every SETS-th unit of the block; warp 4j + r owns tile r (rows
//    32r..32r+31) and keeps its own cp.async.bulk ring of that tile's units.
//    Per group of 32 columns it writes the exact integer weights c - z as a
//    BF16 A operand (128 rows x 32 columns) into a TMEM buffer, and later
//    reads back that group's FP32 product D = (c - z) x from TMEM and adds
//    s * D to its rows' sums.  The outlier columns enter the same way with
//    their BF16 weights and s = 1.
//  * one MMA warp per set, whose elected lane issues two tcgen05.mma
//    kind::f16 (M = 128, N = MB, K = 16) per group into the group's own D
//    buffer.
//
// Groups travel in chunks of H: the compute warps store H groups' A operands
// and arrive once, the MMA lane waits once, issues 2H MMAs and commits once,
// and the compute warps wait once before reading the H D buffers back.  Each
// mbarrier operation costs the issuing thread on the order of a hundred
// cycles, more than one group's two MMAs, so handshakes per group would pace
// the kernel.
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
// Handshakes, per set and chunk slot q (Q slots of H TMEM buffers, used
// round robin): full[q] (one arrival per compute warp, after its TMEM stores
// and x writes) -> MMA issue -> done[q] (tcgen05.commit) -> compute threads
// read the chunk's D buffers.  A slot is rebuilt only after its previous
// chunk was read back, so the MMAs that read its A operands have completed.  Every wait is bounded; a timeout raises the
// device error bit and turns the remaining waits into no-ops.
constexpr int kTcTmemCols = 512;

template <int MB_, int SETS_, int H_, int Q_>
struct TcCfg {
    static constexpr int MB = MB_;
    static constexpr int SETS = SETS_;               // warp sets
    static constexpr int H = H_;                     // groups per handshake (a chunk)
    static constexpr int Q = Q_;                     // chunk slots per set
    static constexpr int P = H * Q;                  // TMEM group buffers per set
    static constexpr int CW = 4 * SETS;              // compute warps
    static constexpr int WARPS = CW + SETS;          // + one MMA warp per set
    static constexpr int DCOL = (SETS * P * 16 + 31) / 32 * 32;  // A buffers below, D from here
    static constexpr int XBYTES = 256 * MB * 2;      // x image of one super-group
    static constexpr int KSTEP = MB * 32;            // bytes of one 16-column K step of x
    static_assert(DCOL + SETS * P * MB <= kTcTmemCols, "TMEM budget");
    static_assert(DCOL % 32 == 0, "D alignment");
    static_assert(H >= 1 && H <= 8 && Q >= 2 && Q <= 8, "chunk shape");
};

// 16 rows: three sets of four compute warps (four warps per sub-partition
// keep each thread within 128 registers), chunks of two groups, two chunk
// slots per set.  32 rows: the D buffers are twice as wide, so two sets.
using TcCfg16 = TcCfg<16, 3, 2, 2>;
using TcCfg32 = TcCfg<32, 2, 2, 2>;

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

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
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
        const uint32_t sa = smem_u32(stage);
        const uint4 q = lds128(sa + g * 512 + lane * 16);
        const uint32_t sw = lds32(sa + 4096 + lane * 16 + (g >> 1) * 4);
        const uint32_t zw = lds32(sa + 4608 + lane * 4);
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

template <typename C>
__global__ void __launch_bounds__(C::WARPS * 32, 1) gemm_tc_kernel(const TcArgs args) {
    constexpr int MB = C::MB;
    extern __shared__ __align__(1024) uint8_t tsm[];
    const Prob &a = args.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cr = (a.cl > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int D = args.depth;
    // shared memory: [x images SETS x 2][ring CW x D]
    // [bars][tmem slot, abort].  At a block end, once every group of the block
    // has been read back, set j's first x image holds its 128 x MB partial
    // sums (the same 256 x MB x 2 bytes).
    uint8_t *ximg = tsm;
    uint8_t *ring_base = ximg + (size_t)C::SETS * 2 * C::XBYTES;
    auto red_of = [&](int set) { return reinterpret_cast<float *>(ximg + (size_t)set * 2 * C::XBYTES); };
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring_base + (size_t)C::CW * D * kStageBytes);
    uint64_t *full = bars + C::CW * D;      // [SETS][Q]
    uint64_t *done = full + C::SETS * C::Q;  // [SETS][Q]
    uint64_t *fin = done + C::SETS * C::Q;   // [SETS]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + C::SETS);
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
        for (int b = 0; b < C::SETS * C::Q; ++b) {
            mbar_init(smem_u32(&full[b]), 4u);  // one arrival per compute warp of the set
            mbar_init(smem_u32(&done[b]), 1u);
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

        // Two chunk slots: the chunk built last is read back right after the
        // next one is built, so one chunk is in the MMA while the warp builds
        // the next.  When a unit starts, every chunk of the unit before the
        // previous one has been read back, so the MMAs that read the x image
        // about to be rewritten have completed.
        static_assert(C::Q == 2, "two chunk slots");
        int ci = 0, xl = 0;
        int pnh = 0;       // groups of the pending chunk (0: none)
        float ps[C::H];    // their scales
        float y[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) y[m] = 0.f;
#pragma unroll
        for (int h = 0; h < C::H; ++h) ps[h] = 0.f;
        // read back the pending chunk (built as chunk ci - 1, slot (ci - 1) & 1)
        auto read_back = [&]() {
            const int q = (ci - 1) & 1;
            // every lane waits: no divergent branch around the wait
            tc_wait(smem_u32(&donej[q]), (uint32_t)((ci - 1) >> 1) & 1u, abort);
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int h = 0; h < C::H; ++h) {
                if (h < pnh) {  // warp-uniform
                    const uint32_t td = tl + (uint32_t)(C::DCOL + (j * C::P + q * C::H + h) * MB);
                    const float2 s2 = make_float2(ps[h], ps[h]);
#pragma unroll
                    for (int hh = 0; hh < MB / 16; ++hh) {
                        float dv[16];
                        tmem_ld_d<16>(td + 16 * hh, dv);
#pragma unroll
                        for (int m = 0; m < 16; m += 2) {
                            const float2 r2 = __ffma2_rn(s2, make_float2(dv[m], dv[m + 1]),
                                                         make_float2(y[16 * hh + m], y[16 * hh + m + 1]));
                            y[16 * hh + m] = r2.x;
                            y[16 * hh + m + 1] = r2.y;
                        }
                    }
                }
            }
            pnh = 0;
        };

        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride) {
            const int t = 4 * blk + r;
            const bool active = t < a.T;
            for (int lu = j; lu < nunits; lu += C::SETS, ++xl) {
                const int u = tc_unit(a, sg0, nsg, ob0, lu);
                uint8_t *xb = ximg + (size_t)(j * 2 + (xl & 1)) * C::XBYTES;
                tc_store_x<MB>(a, u, tid, xp, xb);
                if (xblk < args.nblk) {
                    tc_load_x<MB>(a, tc_unit(a, sg0, nsg, ob0, xlu), tid, xp);
                    advance(xblk, xlu);
                }
                const uint8_t *stage = nullptr;
                if (active) stage = ring_acquire(ring, lane);
                else ring_advance_consume(ring);
                __syncwarp();
                const int ngr = tc_groups(a, u);
                for (int g0 = 0; g0 < ngr; g0 += C::H) {
                    // one chunk: up to H groups' A operands, then one arrival
                    const int q = ci & 1;
                    const int nh = min(C::H, ngr - g0);
                    float sc[C::H];
#pragma unroll
                    for (int h = 0; h < C::H; ++h) {
                        sc[h] = 0.f;
                        if (h < nh) {  // warp-uniform
                            uint32_t av[16];
                            sc[h] = tc_build_a(a, u, g0 + h, stage, lane, av);
                            tmem_st16(tl + (uint32_t)((j * C::P + q * C::H + h) * 16), av);
                        }
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&fullj[q]));
                    if (pnh) read_back();
                    ++ci;
                    pnh = nh;
#pragma unroll
                    for (int h = 0; h < C::H; ++h) ps[h] = sc[h];
                }
                if (active) ring_release(ring);
                if (iblk < args.nblk) {
                    const int ti = 4 * iblk + r;
                    if (ti < a.T) ring_issue(ring, a, ti, tc_unit(a, sg0, nsg, ob0, ilu), lane);
                    else ring_advance_issue(ring);
                    advance(iblk, ilu);
                }
            }
            if (pnh) read_back();
            // block end: sets 1.. hand their sums to set 0 (each set's own x
            // image is free: its groups are all read back), which adds them in
            // set order and stores the rows (or, in a cluster, leaves them for
            // the rank-ordered reduction)
            if (j > 0) {
                float *red = red_of(j);
#pragma unroll
                for (int m = 0; m < MB; ++m) red[(32 * r + lane) * MB + m] = y[m];
            }
            named_sync(1, 32 * C::CW);
            if (j == 0) {
                for (int o = 1; o < C::SETS; ++o) {
                    const float *red = red_of(o);
#pragma unroll
                    for (int m = 0; m < MB; ++m) y[m] += red[(32 * r + lane) * MB + m];
                }
                if (a.cl > 1) {
                    float *red = red_of(0);
#pragma unroll
                    for (int m = 0; m < MB; ++m) red[(32 * r + lane) * MB + m] = y[m];
                } else if (active) {
#pragma unroll
                    for (int m = 0; m < MB; ++m) store_y(a, t, lane, m, y[m]);
                }
            }
            named_sync(1, 32 * C::CW);
#pragma unroll
            for (int m = 0; m < MB; ++m) y[m] = 0.f;
        }
        ring_drain(ring);
    } else if (lane == 0) {
        // ------------------------------------------------ MMA issuer of set j (one lane)
        const int j = warp - C::CW;
        pdl_wait();
        const uint32_t idesc = bf16_idesc<MB>();
        int q = 0, xl = 0;
        bool any = false;
        for (int blk = blockIdx.x / a.cl; blk < args.nblk; blk += bstride) {
            for (int lu = j; lu < nunits; lu += C::SETS, ++xl) {
                const int ngr = tc_groups(a, tc_unit(a, sg0, nsg, ob0, lu));
                const uint32_t xs0 = smem_u32(ximg + (size_t)(j * 2 + (xl & 1)) * C::XBYTES);
                for (int g0 = 0; g0 < ngr; g0 += C::H, ++q) {
                    const int sl = q % C::Q;
                    const int nh = min(C::H, ngr - g0);
                    const bool ok = tc_wait(smem_u32(&full[j * C::Q + sl]), (uint32_t)(q / C::Q) & 1u, abort);
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (ok) {
                        for (int h = 0; h < nh; ++h) {
                            const int b = sl * C::H + h;
                            const uint32_t xs = xs0 + (uint32_t)(2 * (g0 + h) * C::KSTEP);
                            const uint32_t ta = tmem + (uint32_t)((j * C::P + b) * 16);
                            const uint32_t td = tmem + (uint32_t)(C::DCOL + (j * C::P + b) * MB);
#pragma unroll
                            for (int k = 0; k < 2; ++k) {
                                const uint64_t bdesc = umma_desc(xs + (uint32_t)(k * C::KSTEP), 128u, 256u);
                                asm volatile(
                                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
                                    "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(td),
                                    "r"(ta + 8u * k), "l"(bdesc), "r"((uint32_t)k), "r"(idesc)
                                    : "memory");
                            }
                        }
                        any = true;
                    }
                    // one commit per chunk: done[sl] fires when all its MMAs completed
                    asm volatile(
                        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                            smem_u32(&done[j * C::Q + sl]))
                        : "memory");
                }
            }
        }
        // every MMA this lane issued has completed before TMEM is released
        if (any) {
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    smem_u32(&fin[j]))
                : "memory");
            tc_wait(smem_u32(&fin[j]), 0u, abort);
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
                const float *rp = cluster.map_shared_rank(red_of(0), rk) + (32 * warp + lane) * MB;
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

template <typename C>
size_t tc_smem_bytes(int depth) {
    return (size_t)C::SETS * 2 * C::XBYTES + (size_t)C::CW * depth * kStageBytes +
           (size_t)(C::CW * depth + 2 * C::SETS * C::Q + C::SETS) * 8 + 16;
}

template <typename C>
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
    int depth = 2;  // two units in flight per warp; a third measured slower (shared memory left to L1)
    while (depth > 1 && tc_smem_bytes<C>(depth) > dev.smem_optin) --depth;
    args.depth = depth;
    const size_t smem = tc_smem_bytes<C>(depth);
    if (smem > dev.smem_optin) return SPECTRA_ERR_SHAPE;
    cudaError_t e = prepare_kernel(gemm_tc_kernel<C>, done, dev);
    if (e != cudaSuccess) return SPECTRA_ERR_CUDA;
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

spectra_status tc_device_error(bool *raised, cudaStream_t s) {
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

}  // namespace spectra
