// Device math shared by the kernels of libssd.so.
#pragma once

#include <cuda_runtime.h>

namespace ssd {

// softplus for the decay steps, whose time the accurate expf and log1pf bounded:
// softplus(x) = max(x, 0) + log1p(u), u = exp(-|x|) in (0, 1], with u from
// the hardware base-2 exponential (ex2.approx, relative error about 2^-22;
// u below 2^-126 flushes to zero, where softplus(x) = x or 0 to float
// precision anyway) and log1p(u) = u p(u), p the degree-8 Chebyshev
// interpolant of log1p(u)/u on [0, 1] (coefficients from
// mamba_ssd_sequence_b200/gen_log1p_poly.py; relative error 2.6e-7 in float32).
__device__ __forceinline__ float softplus_fast(float x) {
    float u;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(u) : "f"(-fabsf(x) * 1.4426950408889634f));
    float p = 5.126102362e-03f;
    p = fmaf(p, u, -2.907406539e-02f);
    p = fmaf(p, u, 7.751608640e-02f);
    p = fmaf(p, u, -1.360224783e-01f);
    p = fmaf(p, u, 1.907688081e-01f);
    p = fmaf(p, u, -2.483539879e-01f);
    p = fmaf(p, u, 3.331812024e-01f);
    p = fmaf(p, u, -4.999944568e-01f);
    p = fmaf(p, u, 9.999999404e-01f);
    return fmaxf(x, 0.0f) + u * p;
}

// SiLU of a convolution output, u / (1 + e^-u) with the fast exponential and
// division.  The standalone convolution and the one fused into the order-1
// chunk-state kernel both use it, so the two give the same bits.
__device__ __forceinline__ float silu_fast(float u) { return __fdividef(u, 1.0f + __expf(-u)); }

}  // namespace ssd
