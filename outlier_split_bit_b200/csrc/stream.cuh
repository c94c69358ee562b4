// stream.cuh -- the weight-streaming machinery shared by the matvec kernels
// (gemv.cu) and the tensor-core kernel (gemm_tc.cu): the kernels' view of one
// problem, the RT32 unit copies into per-warp shared-memory rings (cp.async.bulk
// completing on mbarriers, with bounded waits), the code decoder's pairing,
// and the host launch helpers.  Everything here has internal linkage, so each
// translation unit that includes it gets its own copy, including its own
// device error word.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace spectra {
namespace {

constexpr int kOB = 8;                         // outlier octets per unit
constexpr int kSgBytes = 8 * 512 + 512 + 128;  // codes + scales + zeros of a warp per super-group
constexpr int kOctBytes = 512;                 // outlier bytes of a warp per octet
constexpr int kStageBytes = kSgBytes;          // one ring stage (16-byte multiple)
constexpr uint64_t kWaitNs = 1000000000ull;    // a wait gives up after one second (%globaltimer)
constexpr uint32_t kWaitRounds = 1u << 22;      // backstop on try_wait rounds
constexpr uint32_t kSuspendNs = 500000;        // per-round suspend hint (an upper bound only)

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
    const int32_t *bidx;  // bulk column list of a compacted bulk, nullptr when masked
    void *y;
    int n, k, m, G, S, O8, n_o, T;  // k: bulk columns (the geometry of the codes)
    int kx;                         // columns of x (its row stride)
    int U;         // units per tile
    int ppc, tpc;  // slices per tile, tiles per CTA item
    int lgp;       // log2(ppc) where ppc is a power of two (persistent kernel)
    int cl;        // CTAs per cluster (cluster kernel)
    int ytype;
    int items;     // ceil(T / tpc)
};


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

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// One try of phase `parity` of an mbarrier.  The thread sleeps until the
// phase completes or the suspend hint expires (it may also return earlier),
// so waiting warps leave the issue slots to the computing ones.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier.  Bounded by elapsed time: it gives
// up once kWaitNs of %globaltimer time have passed since the first failed
// try (the count of tries is only a backstop, since a try may return before
// its hint expires).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kWaitRounds; ++i) {
        if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
    return false;
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

// BF16 pair (128 + c_s, 128 + c_{s+4}) of nibbles s and s + 4 of a word.
template <int sh>
__device__ __forceinline__ uint32_t code_pair(uint32_t w) {
    return ((w >> (4 * sh)) & 0x000F000Fu) | 0x43004300u;
}

// A load of x.  kL2 = false: through L1 (ld.global.nc), for kernels in which
// no CTA writes x (an earlier launch's output is ordered by the programmatic
// dependency wait).  kL2 = true: at L2 (ld.global.cg), for the chain kernel,
// where x may be the output of an earlier matvec of the same launch, so a
// line cached in L1 before that write would be stale.
template <bool kL2, typename T>
__device__ __forceinline__ T ld_x(const T *p) {
    if constexpr (kL2) return __ldcg(p);
    else return __ldg(p);
}

// x of 8 consecutive columns c0..c0+7 of a compacted bulk for batch row m,
// as 4 BF16 pairs in column order: gathered through the bulk column list,
// padding (and any entry outside [0, kx)) read as +0.  c0 is a multiple of 8.
template <bool kL2 = false>
__device__ __forceinline__ uint4 bulk_x8_gather(const Prob &a, int m, int c0) {
    const uint16_t *xr = a.x + (size_t)m * a.kx;
    const int4 b0 = __ldg(reinterpret_cast<const int4 *>(a.bidx + c0));
    const int4 b1 = __ldg(reinterpret_cast<const int4 *>(a.bidx + c0 + 4));
    const int c[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = ((unsigned)c[e] < (unsigned)a.kx) ? (uint32_t)ld_x<kL2>(xr + c[e]) : 0u;
    return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                      h[6] | (h[7] << 16));
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
    int cslot, islot;  // consumed % D and issued % D, kept incrementally
    uint32_t cphase;   // (consumed / D) & 1
    bool ok;
    int failed_at;
};

__device__ __forceinline__ void ring_init(Ring &r, uint8_t *base, uint64_t *bars, int D, int lane) {
    r.base = base;
    r.base_s = smem_u32(base);
    r.bar_s = smem_u32(bars);
    r.D = D;
    r.consumed = r.issued = 0;
    r.cslot = r.islot = 0;
    r.cphase = 0u;
    r.ok = true;
    r.failed_at = 0;
    if (lane == 0) {
        for (int d = 0; d < D; ++d) mbar_init(r.bar_s + 8u * d, 1u);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
}

// Advance the issue side by one stage (after a copy, or for a unit that is
// skipped on both sides).
__device__ __forceinline__ void ring_advance_issue(Ring &r) {
    if (!r.ok) return;
    ++r.issued;
    if (++r.islot == r.D) r.islot = 0;
}

__device__ __forceinline__ void ring_issue(Ring &r, const Prob &a, int t, int u, int lane) {
    const int d = r.islot;
    if (r.ok && lane == 0)
        issue_unit(a, t, u, r.base_s + (uint32_t)d * kStageBytes, r.bar_s + 8u * d);
    ring_advance_issue(r);
}

// Wait for the next stage to fill; returns its address (nullptr after a failure).
__device__ __forceinline__ const uint8_t *ring_acquire(Ring &r, int lane) {
    const int d = r.cslot;
    if (r.ok && !mbar_wait(r.bar_s + 8u * d, r.cphase)) {
        r.ok = false;
        r.failed_at = r.consumed;
        if (lane == 0) atomicOr(&g_device_error, 1u);
    }
    return r.ok ? r.base + (size_t)d * kStageBytes : nullptr;
}

// Advance the consume side by one stage.
__device__ __forceinline__ void ring_advance_consume(Ring &r) {
    if (!r.ok) return;
    ++r.consumed;
    if (++r.cslot == r.D) {
        r.cslot = 0;
        r.cphase ^= 1u;
    }
}

__device__ __forceinline__ void ring_release(Ring &r) {
    __syncwarp();
    ring_advance_consume(r);
}

// After a failed wait, let the copies already in flight land before the CTA
// releases its shared memory (bounded as well).
__device__ __forceinline__ void ring_drain(const Ring &r) {
    if (r.ok) return;
    for (int n = r.failed_at; n < r.issued; ++n)
        mbar_wait(r.bar_s + 8u * (n % r.D), (uint32_t)(n / r.D) & 1u);
}

// ---------------------------------------------------------------- host helpers

int units_of(const Geometry &g) { return g.S + (int)cdiv(g.O8, kOB); }

void fill_prob(Prob &a, const spectra_layer &l, const Geometry &g, const uint16_t *x, int mc,
               void *y, int ytype) {
    a.codes = reinterpret_cast<const uint4 *>(l.codes);
    a.scales = reinterpret_cast<const uint4 *>(l.scales);
    a.zeros = l.zeros;
    a.outw = reinterpret_cast<const uint4 *>(l.outlier_w);
    a.oidx = l.outlier_idx;
    a.x = x;
    a.bidx = l.bulk_idx;
    a.y = y;
    a.n = l.n;
    a.k = g.k;
    a.kx = l.k;
    a.m = mc;
    a.G = g.G;
    a.S = g.S;
    a.O8 = g.O8;
    a.n_o = g.n_o;
    a.T = g.T;
    a.U = units_of(g);
    a.ppc = 1;
    a.tpc = 1;
    a.lgp = 0;
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

}  // namespace
}  // namespace spectra
