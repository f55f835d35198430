// Device helpers shared by the two tensor-core convolution kernels (k_back_conv_tc.cu: tap shifts;
// k_back_conv_tcn.cu: taps in the N dimension): per-row window geometry, exact small divisions and reductions.
#pragma once
#include "vf_internal.cuh"

namespace vf {
namespace conv_tc {

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Per row of a group: the origins of its windows on their maps (ay * y_j + by, ax * x_j + bx) for wa and wd,
// its centre and its coefficient row. Computed once per group into shared memory.
struct RowGeo {
    int aoy, aox, doy, dox;
    long long b;
    const float* arow;
};

// P: any parameter block with members A (RowRef), pg (PassGeom), ps (PassStart), wa and wd (Win).
template <class P>
__device__ __forceinline__ RowGeo row_geo(const P& p, long long m) {
    const long long gl = p.pg.pass_m0 + m;
    float sg;
    const long long j = start_neuron(p.pg, p.ps.n, m, &sg);
    const int xj = (int)(j % p.ps.w);
    const int yj = (int)((j / p.ps.w) % p.ps.h);
    RowGeo r;
    r.aoy = p.wa.ay * yj + p.wa.by;
    r.aox = p.wa.ax * xj + p.wa.bx;
    r.doy = p.wd.ay * yj + p.wd.by;
    r.dox = p.wd.ax * xj + p.wd.bx;
    r.b = gl / p.pg.R_pass;
    r.arow = p.A.row(m);
    return r;
}

// n / d for 0 <= n < 2^22 and d >= 1, exact: (n + 0.5) / d is at least 1/(2d) from an integer, further than
// the rounding of (n + 0.5) * (1/d) in fp32 can move it.
__device__ __forceinline__ int fdiv(int n, float inv) { return __float2int_rz(((float)n + 0.5f) * inv); }

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

}  // namespace conv_tc
}  // namespace vf
