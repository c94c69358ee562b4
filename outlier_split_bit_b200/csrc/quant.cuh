// quant.cuh -- the Group-32 4-bit quantiser of one group, in IEEE double
// (shared by the weight packer and the KV-cache append).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: Group-32 4-bit codes
// with a scale and a bit-packed zero point per group.  Per group of 32
// values v (read with -0 as +0): lo = min, hi = max; the FP16 scale is
// (hi - lo) / 15 rounded once to nearest even; with S its value, z =
// clamp(rint(-lo / S), 0, 15) and c = clamp(rint(v / S) + z, 0, 15), every
// division an IEEE double division (__ddiv_rn and friends are never
// contracted into FMA), rint rounding half to even; S == 0 gives z = 0 and
// all codes 0.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace spectra {

__device__ __forceinline__ double clamp015(double v) {
    return v < 0.0 ? 0.0 : (v > 15.0 ? 15.0 : v);
}

// Quantises one group: the FP16 scale bits, the zero point and the 16-byte
// code record (word w, nibble j = code of value 8w + j).  Returns false when
// the scale rounds to FP16 infinity; the record and zero point are then 0.
// With skip_codes the codes are not computed (the record stays 0).
__device__ __forceinline__ bool quantize_group32(const double v[32], uint32_t rec[4],
                                                 unsigned short *scale_bits, uint32_t *zero,
                                                 bool skip_codes = false) {
    double lo = v[0], hi = v[0];
#pragma unroll
    for (int kk = 1; kk < 32; ++kk) {
        if (v[kk] < lo) lo = v[kk];
        if (v[kk] > hi) hi = v[kk];
    }
    const double q15 = __ddiv_rn(__dsub_rn(hi, lo), 15.0);
    unsigned short hbits;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(hbits) : "d"(q15));
    *scale_bits = hbits;
    *zero = 0;
    const bool finite = (hbits & 0x7FFFu) != 0x7C00u;
    const double Sd = (double)__half2float(__ushort_as_half(hbits));
    if (Sd != 0.0 && finite && !skip_codes) {
        const double zd = clamp015(rint(__ddiv_rn(-lo, Sd)));
        *zero = (uint32_t)zd;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            const double c = clamp015(__dadd_rn(rint(__ddiv_rn(v[kk], Sd)), zd));
            rec[kk >> 3] |= (uint32_t)c << (4 * (kk & 7));
        }
    }
    return finite;
}

}  // namespace spectra
