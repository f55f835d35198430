// Sound-in-fp32 bounds: rounding-error budgets for the verify path.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §4.2 (soundness is a one-sided over-approximation) and §1 (bounds for
// every input of the domain). The page says nothing on floating point; these kernels make the fp32 path
// one-sided without it, on this library's own error analysis:
//
//   * every FFMA dot product of K terms errs by at most gamma_K = K u / (1 - K u) times the sum of the
//     terms' magnitudes (u = 2^-24, any summation order), so interval propagation widens each radius by
//     gamma times |W| (|c| + r) + |b|, and ends are rounded outwards;
//   * a back-substituted row errs, at each node v it passes, by at most sum_i |lambda_v,i| w_v,i, where
//     lambda_v are the row's coefficients over v (as computed) and w_v the node's rounding weights:
//     contraction through an affine node gamma_Kb |W| M_src (M: a magnitude bound of the node's value over
//     the box), its bias gamma_N |b|; the relaxation product at a ReLU u M_z, its intercept gamma_N t;
//     the concretisation at the input gamma (|c| + eps); a sum of rows from several consumers u M_v. The
//     executor subtracts that budget from each row's constant as the row passes the node (row_budget_k),
//     rounding down, so every pass's lower bound already holds in exact arithmetic;
//   * the upper ReLU relaxation is made valid in fp32 by rounding its intercept up at both ends.
#include <math.h>

#include "vf_internal.cuh"

namespace vf {

namespace {

constexpr float kU = 0x1p-23f;  // unit roundoff 2^-24, doubled to absorb the (1 + u) factors of each step

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

#define SGRID(i, n) \
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (n); i += (long long)gridDim.x * blockDim.x)

// zr <- zr + g * (S + |b|), rounded up (S = |W| (|c| + r) of the same affine node).
__global__ void sound_radius_k(float* __restrict__ zr, const float* __restrict__ S, const float* __restrict__ bias,
                               long long total, long long n, long long per_channel, float g) {
    SGRID(i, total) {
        const float b = fabsf(bias[(i % n) / per_channel]);
        zr[i] = __fadd_ru(zr[i], __fmul_ru(g, __fadd_ru(S[i], b)));
    }
}

// T = |c| + r, rounded up.
__global__ void abs_plus_k(const float* __restrict__ c, const float* __restrict__ r, long long total,
                           float* __restrict__ T) {
    SGRID(i, total) T[i] = __fadd_ru(fabsf(c[i]), r[i]);
}

// ReLU of [c - r, c + r] with the ends rounded outwards; the result's centre is the rounded midpoint and
// its radius the larger distance to either end, rounded up, so the new interval holds the exact one.
__global__ void sound_relu_k(const float* __restrict__ c, const float* __restrict__ r, long long total,
                             const signed char* __restrict__ split, float* __restrict__ oc, float* __restrict__ orad) {
    SGRID(i, total) {
        float lo = fmaxf(__fsub_rd(c[i], r[i]), 0.f);
        float hi = fmaxf(__fadd_ru(c[i], r[i]), 0.f);
        if (split != nullptr && split[i] < 0) lo = hi = 0.f;
        const float m = __fmul_rn(0.5f, __fadd_rn(lo, hi));
        oc[i] = m;
        orad[i] = fmaxf(__fsub_ru(m, lo), __fsub_ru(hi, m));
    }
}

// Sum of two intervals: the centre's rounding error is recovered exactly (two-sum) and added to the
// radius, rounded up.
__global__ void sound_add_k(const float* __restrict__ c1, const float* __restrict__ r1, const float* __restrict__ c2,
                            const float* __restrict__ r2, long long total, float* __restrict__ oc,
                            float* __restrict__ orad) {
    SGRID(i, total) {
        const float a = c1[i], b = c2[i];
        const float s = __fadd_rn(a, b);
        const float bb = __fsub_rn(s, a);
        const float e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
        oc[i] = s;
        orad[i] = __fadd_ru(__fadd_ru(r1[i], r2[i]), fabsf(e));
    }
}

// Magnitude bounds: M = max(|l|, |u|) (pos_only: max(u, 0), the output of a ReLU over [l, u]).
__global__ void magnitude_k(const float* __restrict__ l, const float* __restrict__ u, long long total, int pos_only,
                            float* __restrict__ M) {
    SGRID(i, total) M[i] = pos_only ? fmaxf(u[i], 0.f) : fmaxf(fabsf(l[i]), fabsf(u[i]));
}

// Input node: w = g0 (|c| + eps).
__global__ void input_weight_k(const float* __restrict__ c, float eps, long long total, float g0,
                               float* __restrict__ w) {
    SGRID(i, total) w[i] = __fmul_ru(g0, __fadd_ru(fabsf(c[i]), eps));
}

// Affine node, in place over Q = fl(|W| M_src): w = gQ Q + gN |b| + u M_v, rounded up (gQ includes the
// factor for Q's own rounding). Mv may be null.
__global__ void affine_weight_k(float* __restrict__ w, const float* __restrict__ bias, const float* __restrict__ Mv,
                                long long total, long long n, long long per_channel, float gQ, float gN) {
    SGRID(i, total) {
        const float b = fabsf(bias[(i % n) / per_channel]);
        float a = __fadd_ru(__fmul_ru(gQ, w[i]), __fmul_ru(gN, b));
        if (Mv != nullptr) a = __fadd_ru(a, __fmul_ru(kU, Mv[i]));
        w[i] = a;
    }
}

// ReLU node: w = 2u M_z + gN t (the relaxation product, a sum at the output, the intercept), rounded up.
__global__ void relu_weight_k(const float4* __restrict__ P, const float* __restrict__ l, const float* __restrict__ u,
                              long long total, float gN, float* __restrict__ w) {
    SGRID(i, total) {
        const float mz = fmaxf(fabsf(l[i]), fabsf(u[i]));
        w[i] = __fadd_ru(__fmul_ru(2.f * kU, mz), __fmul_ru(gN, P[i].z));
    }
}

// Other nodes (add): w = u M_v.
__global__ void scale_up_k(const float* __restrict__ M, long long total, float g, float* __restrict__ w) {
    SGRID(i, total) w[i] = __fmul_ru(g, M[i]);
}

// cst[m] -= sum_j |x_j| w[b, j] for the rows over one node (relaxed by rx first when given), the sum rounded
// up and the difference down. One CTA per row.
__global__ void __launch_bounds__(256)
row_budget_k(RowRef A, Relax rx, long long M, int n, PassGeom pg, const float* __restrict__ w,
             float* __restrict__ cst) {
    __shared__ float red[8];
    for (long long m = blockIdx.x; m < M; m += gridDim.x) {
        const float* a = A.row(m);
        const long long b = (pg.pass_m0 + m) / pg.R_pass;
        float acc = 0.f;
        for (int j = threadIdx.x; j < n; j += 256) {
            float x = fabsf(a[j]);
            if (rx.P != nullptr) {
                const float4 p = rx.P[b * n + j];
                x = __fmul_ru(x, a[j] >= 0.f ? p.x : p.y);
            }
            acc = __fmaf_ru(x, w[b * n + j], acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc = __fadd_ru(acc, __shfl_xor_sync(0xffffffffu, acc, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.f;
            for (int k = 0; k < 8; ++k) t = __fadd_ru(t, red[k]);
            cst[m] = __fsub_rd(cst[m], t);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_sound_radius(float* zr, const float* S, const float* bias, long long total, long long n,
                                long long per_channel, float g, cudaStream_t s) {
    sound_radius_k<<<grid_for(total, 256), 256, 0, s>>>(zr, S, bias, total, n, per_channel, g);
    return cudaGetLastError();
}

cudaError_t launch_abs_plus(const float* c, const float* r, long long total, float* T, cudaStream_t s) {
    abs_plus_k<<<grid_for(total, 256), 256, 0, s>>>(c, r, total, T);
    return cudaGetLastError();
}

cudaError_t launch_sound_relu(const float* c, const float* r, long long total, const signed char* split, float* oc,
                              float* orad, cudaStream_t s) {
    sound_relu_k<<<grid_for(total, 256), 256, 0, s>>>(c, r, total, split, oc, orad);
    return cudaGetLastError();
}

cudaError_t launch_sound_add(const float* c1, const float* r1, const float* c2, const float* r2, long long total,
                             float* oc, float* orad, cudaStream_t s) {
    sound_add_k<<<grid_for(total, 256), 256, 0, s>>>(c1, r1, c2, r2, total, oc, orad);
    return cudaGetLastError();
}

cudaError_t launch_magnitude(const float* l, const float* u, long long total, int pos_only, float* M, cudaStream_t s) {
    magnitude_k<<<grid_for(total, 256), 256, 0, s>>>(l, u, total, pos_only, M);
    return cudaGetLastError();
}

cudaError_t launch_input_weight(const float* c, float eps, long long total, float g0, float* w, cudaStream_t s) {
    input_weight_k<<<grid_for(total, 256), 256, 0, s>>>(c, eps, total, g0, w);
    return cudaGetLastError();
}

cudaError_t launch_affine_weight(float* w, const float* bias, const float* Mv, long long total, long long n,
                                 long long per_channel, float gQ, float gN, cudaStream_t s) {
    affine_weight_k<<<grid_for(total, 256), 256, 0, s>>>(w, bias, Mv, total, n, per_channel, gQ, gN);
    return cudaGetLastError();
}

cudaError_t launch_relu_weight(const float4* P, const float* l, const float* u, long long total, float gN, float* w,
                               cudaStream_t s) {
    relu_weight_k<<<grid_for(total, 256), 256, 0, s>>>(P, l, u, total, gN, w);
    return cudaGetLastError();
}

cudaError_t launch_scale_up(const float* M, long long total, float g, float* w, cudaStream_t s) {
    scale_up_k<<<grid_for(total, 256), 256, 0, s>>>(M, total, g, w);
    return cudaGetLastError();
}

cudaError_t launch_row_budget(const RowRef& A, Relax rx, long long M, int n, PassGeom pg, const float* w, float* cst,
                              cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    long long g = M < 148LL * 16 ? M : 148LL * 16;
    row_budget_k<<<(unsigned)g, 256, 0, s>>>(A, rx, M, n, pg, w, cst);
    return cudaGetLastError();
}

// gamma_K = K u / (1 - K u), u = 2^-24, rounded up to a float.
float gamma_up(long long K) {
    const double u = ldexp(1.0, -24);
    const double g = (double)K * u / (1.0 - (double)K * u);
    return nextafterf((float)g, INFINITY);
}

}  // namespace vf
