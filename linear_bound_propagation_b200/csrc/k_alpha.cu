// alpha-CROWN: per-row lower ReLU slopes for the specification bound, their gradient and the Adam
// ascent step.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (alpha-CROWN among the bound-propagation methods) and §3 / §4.3
// (the per-neuron alpha tensors, i.e. the lower ReLU slopes, that alpha-CROWN optimises).
//
// For a specification row the bound is a function of the lower slopes of the unstable neurons
// (0 < up < 1). Back-substitution applies, at each ReLU, lam_z = slope * lam_h with slope = alpha for
// lam_h >= 0 (unstable neurons) and the intercept term min(lam_h, 0) * t. Its gradient runs the chain in
// the other direction: at the input G = c - eps * sign(lam_in); through a dense node G_z = G_h W^T + b;
// at a ReLU d lb / d alpha_i = G_z,i * lam_h,i for lam_h,i >= 0 (unstable i), and
// G_h = G_z * slope + [lam_h < 0] * t.
//
// Split constraints (beta-CROWN with branch-and-bound, same page §2.2 and §4.3): on a subdomain where
// s_i z_i >= 0, lb may add -beta_i s_i z_i for any beta_i >= 0, so lam_z gains -beta_i s_i at the ReLU;
// d lb / d beta_i = -s_i G_z,i, and beta takes the same Adam step, projected to beta >= 0.
#include <math.h>

#include "vf_internal.cuh"

namespace vf {

namespace {

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

__device__ __forceinline__ bool unstable(const float4& p) { return p.y > 0.f && p.y < 1.f; }

// Z[m, :] (=, += with accumulate) slope * H[m, :] with per-row slopes for unstable neurons (alpha ==
// nullptr: the table's own lower slope); cst[m] += sum min(H, 0) * t (+ Z * bias, bias in P.w, when
// with_bias). One warp per row: each lane takes four columns 32 apart per step, so a warp's loads of a
// step cover 4 x 128 contiguous bytes and are all issued before they are used; a warp reduction gives the
// row constant.
__global__ void __launch_bounds__(256)
relax_alpha_rows_k(const float* __restrict__ H, long long M, int n, const float4* __restrict__ P, PassGeom pg,
                   const float* __restrict__ alpha, float* __restrict__ Z, float* __restrict__ cst, int with_bias,
                   int accumulate, const signed char* __restrict__ split, const float* __restrict__ beta) {
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const long long b = (pg.pass_m0 + m) / pg.R_pass;
        const float* h = H + m * n;
        const float* al = alpha != nullptr ? alpha + m * n : nullptr;
        const float* be = beta != nullptr ? beta + m * n : nullptr;
        const float4* Pb = P + b * n;
        const signed char* sp = split != nullptr ? split + b * n : nullptr;
        float* z = Z + m * n;
        float cs = 0.f;
        for (int i0 = lane; i0 < n; i0 += 128) {
            float x[4], a[4], old[4], bv[4];
            float4 p[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                const bool in = i < n;
                x[u] = in ? h[i] : 0.f;
                p[u] = in ? Pb[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                a[u] = (in && al != nullptr) ? al[i] : 0.f;
                old[u] = (in && accumulate) ? z[i] : 0.f;
                bv[u] = (in && be != nullptr && sp != nullptr && sp[i] != 0) ? (float)sp[i] * be[i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                if (i >= n) break;
                const float lo = (al != nullptr && unstable(p[u])) ? a[u] : p[u].x;
                const float r = ((x[u] >= 0.f) ? x[u] * lo : x[u] * p[u].y) - bv[u];
                cs = fmaf(fminf(x[u], 0.f), p[u].z, cs);
                if (with_bias) cs = fmaf(r, p[u].w, cs);
                z[i] = accumulate ? old[u] + r : r;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
        if (lane == 0) cst[m] += cs;
    }
}

// lb[m] = cst[m] + lam . c - eps |lam|_1 and G[m, i] = c_i - eps * sign(lam_i). One warp per row.
__global__ void __launch_bounds__(256)
concretize_grad_k(const float* __restrict__ lam, long long M, int n0, PassGeom pg, const float* __restrict__ centres,
                  float eps, const float* __restrict__ cst, float* __restrict__ lb, float* __restrict__ G) {
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const float* a = lam + m * n0;
        const float* c = centres + ((pg.pass_m0 + m) / pg.R_pass) * (long long)n0;
        float s = 0.f;
        for (int i = lane; i < n0; i += 32) {
            const float x = a[i];
            s += fmaf(x, c[i], -eps * fabsf(x));
            if (G != nullptr) G[m * n0 + i] = c[i] - eps * ((x > 0.f) ? 1.f : ((x < 0.f) ? -1.f : 0.f));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) lb[m] = s + cst[m];
    }
}

// Through one ReLU of the chain, in place: g = d lb / d alpha (unstable, lam_h >= 0), then
// G <- G * slope + [H < 0] * t (slope from the current alpha), then (adam_step > 0) one Adam ascent step
// on alpha, projected to [0, 1]. grad_out (optional) receives g.
__device__ __forceinline__ float adam_ascent(float x, float g, float* m1, float* m2, float lr, float c1, float c2) {
    const float v1 = 0.9f * *m1 + 0.1f * g;
    const float v2 = 0.999f * *m2 + 0.001f * g * g;
    *m1 = v1;
    *m2 = v2;
    return x + lr * (v1 * c1) / (sqrtf(v2 * c2) + 1e-8f);
}

// One warp per row, four columns 32 apart per lane and step (the row's centre, and so its relaxation and
// split row, is found once per row rather than by a division per element).
__global__ void __launch_bounds__(256)
relax_grad_adam_k(float* __restrict__ G, const float* __restrict__ H, long long M, int n,
                  const float4* __restrict__ P, PassGeom pg, float* __restrict__ alpha,
                  float* __restrict__ grad_out, float* __restrict__ m1, float* __restrict__ m2,
                  int adam_step, float lr, float c1, float c2, BetaRows bt) {
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const long long b = (pg.pass_m0 + m) / pg.R_pass;
        const float4* Pb = P + b * n;
        const signed char* sp = bt.split != nullptr ? bt.split + b * n : nullptr;
        const long long r0 = m * n;
        for (int i0 = lane; i0 < n; i0 += 128) {
            float x[4], gz[4], a[4];
            float4 p[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                const bool in = i < n;
                p[u] = in ? Pb[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                x[u] = in ? H[r0 + i] : 0.f;
                gz[u] = in ? G[r0 + i] : 0.f;
                a[u] = (in && alpha != nullptr) ? alpha[r0 + i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                if (i >= n) break;
                const long long e = r0 + i;
                const bool un = unstable(p[u]);
                const float al = (alpha != nullptr && un) ? a[u] : p[u].x;
                const float g = (un && x[u] >= 0.f) ? gz[u] * x[u] : 0.f;
                G[e] = gz[u] * ((x[u] >= 0.f) ? al : p[u].y) + ((x[u] < 0.f) ? p[u].z : 0.f);
                if (grad_out != nullptr) grad_out[e] = g;
                if (adam_step > 0 && un && alpha != nullptr)
                    alpha[e] = fminf(fmaxf(adam_ascent(al, g, &m1[e], &m2[e], lr, c1, c2), 0.f), 1.f);
                if (sp != nullptr) {
                    const signed char sg = sp[i];
                    const float gb = (sg != 0) ? -(float)sg * gz[u] : 0.f;
                    if (bt.grad_out != nullptr) bt.grad_out[e] = gb;
                    if (adam_step > 0 && sg != 0 && bt.beta != nullptr)
                        bt.beta[e] = fmaxf(adam_ascent(bt.beta[e], gb, &bt.m1[e], &bt.m2[e], lr, c1, c2), 0.f);
                }
            }
        }
    }
}

// a = max(init, 0) (or 0 without init), b = c = 0: split multipliers and their Adam moments at the start.
__global__ void zero3_k(float* __restrict__ a, float* __restrict__ b, float* __restrict__ c, long long count,
                        const float* __restrict__ init) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < count;
         e += (long long)gridDim.x * blockDim.x) {
        a[e] = init != nullptr ? fmaxf(init[e], 0.f) : 0.f;
        b[e] = 0.f;
        c[e] = 0.f;
    }
}

// alpha[m, i] = P[b, i].x (the adaptive start) and zero Adam moments.
// Start slopes: the relaxation's lower slope, or init[e] clamped to [0, 1] where init is given and init[e] >= 0
// (a negative entry: no start for that entry). Adam's moments start at zero.
__global__ void alpha_init_k(float* __restrict__ alpha, float* __restrict__ m1, float* __restrict__ m2, long long M,
                             int n, const float4* __restrict__ P, PassGeom pg, const float* __restrict__ init) {
    const long long total = M * n;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long m = e / n;
        const float a0 = init != nullptr ? init[e] : -1.f;
        alpha[e] = a0 >= 0.f ? fminf(a0, 1.f) : P[((pg.pass_m0 + m) / pg.R_pass) * n + (e % n)].x;
        m1[e] = 0.f;
        m2[e] = 0.f;
    }
}

__global__ void identity_relax_k(float4* __restrict__ P, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        P[i] = make_float4(1.f, 1.f, 0.f, 0.f);
}

__global__ void best_update_k(float* __restrict__ best, const float* __restrict__ cur, long long M, int first) {
    for (long long m = blockIdx.x * (long long)blockDim.x + threadIdx.x; m < M; m += (long long)gridDim.x * blockDim.x)
        best[m] = first ? cur[m] : fmaxf(best[m], cur[m]);
}

}  // namespace

cudaError_t launch_relax_alpha_rows(const float* H, long long M, int n, const float4* P, PassGeom pg,
                                    const float* alpha, float* Z, float* cst, cudaStream_t s, int with_bias,
                                    int accumulate, BetaRows bt) {
    long long g = (M + 7) / 8;  // eight rows (warps) per CTA
    if (g > 148LL * 16) g = 148LL * 16;
    relax_alpha_rows_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(H, M, n, P, pg, alpha, Z, cst, with_bias, accumulate,
                                                                 bt.split, bt.split != nullptr ? bt.beta : nullptr);
    return cudaGetLastError();
}

cudaError_t launch_concretize_grad(const float* lam, long long M, int n0, PassGeom pg, const float* centres, float eps,
                                   const float* cst, float* lb, float* G, cudaStream_t s) {
    long long g = (M + 7) / 8;
    if (g > 148LL * 16) g = 148LL * 16;
    concretize_grad_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(lam, M, n0, pg, centres, eps, cst, lb, G);
    return cudaGetLastError();
}

cudaError_t launch_relax_grad_adam(float* G, const float* H, long long M, int n, const float4* P, PassGeom pg,
                                   float* alpha, float* grad_out, float* m1, float* m2, int adam_step, float lr,
                                   cudaStream_t s, BetaRows bt) {
    float c1 = 1.f, c2 = 1.f;
    if (adam_step > 0) {
        c1 = 1.f / (1.f - powf(0.9f, (float)adam_step));
        c2 = 1.f / (1.f - powf(0.999f, (float)adam_step));
    }
    long long g = (M + 7) / 8;  // eight rows (warps) per CTA
    if (g > 148LL * 16) g = 148LL * 16;
    relax_grad_adam_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(G, H, M, n, P, pg, alpha, grad_out, m1, m2, adam_step,
                                                                 lr, c1, c2, bt);
    return cudaGetLastError();
}

cudaError_t launch_zero_moments(float* beta, float* m1, float* m2, long long count, cudaStream_t s, const float* init) {
    zero3_k<<<grid_for(count, 256), 256, 0, s>>>(beta, m1, m2, count, init);
    return cudaGetLastError();
}

cudaError_t launch_alpha_init(float* alpha, float* m1, float* m2, long long M, int n, const float4* P, PassGeom pg,
                              cudaStream_t s, const float* init) {
    alpha_init_k<<<grid_for(M * n, 256), 256, 0, s>>>(alpha, m1, m2, M, n, P, pg, init);
    return cudaGetLastError();
}

cudaError_t launch_identity_relax(float4* P, long long n, cudaStream_t s) {
    identity_relax_k<<<grid_for(n, 256), 256, 0, s>>>(P, n);
    return cudaGetLastError();
}

cudaError_t launch_best_update(float* best, const float* cur, long long M, int first, cudaStream_t s) {
    best_update_k<<<grid_for(M, 256), 256, 0, s>>>(best, cur, M, first);
    return cudaGetLastError();
}

}  // namespace vf
