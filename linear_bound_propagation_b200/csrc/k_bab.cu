// Branch and bound over ReLU splits: the per-subdomain decisions, on the device.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.2, §3 and §4.3 (complete verification by beta-CROWN with
// branch-and-bound; the page names the method only).
//
// For every subdomain (one row of a batched bound evaluation): whether its bounds are contradictory
// (some pre-activation l > u: the subdomain holds no input), its lowest row bound, and the neuron to
// split next -- the unstable neuron (l < 0 < u) with the largest intercept of its upper relaxation,
// -u l / (u - l), over all ReLU layers, ties to the first layer and the lowest index.
#include <math.h>

#include "vf_internal.cuh"

namespace vf {

namespace {

// One CTA per subdomain d. The bounds of ReLU layer q's input are pre_lb / pre_ub at
// D * blk_off[q] + d * blk_n[q] (the vf_ibp layout for D centre rows); neuron j of layer q has the
// search-wide index gbase[q] + j.
__global__ void __launch_bounds__(256)
bab_pick_k(const float* __restrict__ pre_lb, const float* __restrict__ pre_ub, int D,
           const long long* __restrict__ blk_off, const int* __restrict__ blk_n, const int* __restrict__ gbase, int nl,
           const float* __restrict__ lb_a, const float* __restrict__ lb_b, int R, BabPick* __restrict__ out) {
    __shared__ float s_sc[8];
    __shared__ int s_ix[8];
    __shared__ int s_empty[8];
    const int d = blockIdx.x;
    float best = -INFINITY;
    int bi = -1;
    int empty = 0;
    for (int q = 0; q < nl; ++q) {
        const int n = blk_n[q];
        const float* L = pre_lb + (long long)D * blk_off[q] + (long long)d * n;
        const float* U = pre_ub + (long long)D * blk_off[q] + (long long)d * n;
        for (int j = threadIdx.x; j < n; j += 256) {
            const float l = L[j], u = U[j];
            if (l > u) empty = 1;
            if (l < 0.f && u > 0.f) {
                const float sc = -u * l / (u - l);
                if (sc > best) {  // j only grows within a thread, so a tie keeps the lower index
                    best = sc;
                    bi = gbase[q] + j;
                }
            }
        }
    }
    // warp then block argmax: larger score, ties to the lower index
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (oi >= 0 && (bi < 0 || os > best || (os == best && oi < bi))) {
            best = os;
            bi = oi;
        }
    }
    const int any_empty = __any_sync(0xffffffffu, empty);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        s_sc[w] = best;
        s_ix[w] = bi;
        s_empty[w] = any_empty;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = s_sc[0];
        int ix = s_ix[0];
        int e = s_empty[0];
        for (int k = 1; k < 8; ++k) {
            e |= s_empty[k];
            if (s_ix[k] >= 0 && (ix < 0 || s_sc[k] > b || (s_sc[k] == b && s_ix[k] < ix))) {
                b = s_sc[k];
                ix = s_ix[k];
            }
        }
        float mn = INFINITY;
        for (int r = 0; r < R; ++r) {
            float v = lb_a[(long long)d * R + r];
            if (lb_b != nullptr) v = fmaxf(v, lb_b[(long long)d * R + r]);
            mn = fminf(mn, v);
        }
        out[d] = BabPick{ix, e, mn, b};
    }
}

__global__ void repeat_row_k(const float* __restrict__ src, long long n, int D, float* __restrict__ dst) {
    const long long total = n * D;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x)
        dst[e] = src[e % n];
}

// x[r, i] = the vertex of the box centre +/- eps where row r's linear lower bound lam[r, :] . x + const is
// smallest: centre - eps where lam > 0, centre + eps where lam < 0, the centre where lam = 0. The fp32 sum or
// difference is rounded towards the centre (__fsub_ru / __fadd_rd), so every point lies inside the box.
__global__ void minimiser_points_k(const float* __restrict__ centre, const float* __restrict__ lam, float eps,
                                   long long n, int R, float* __restrict__ x) {
    const long long total = n * R;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const float c = centre[e % n], l = lam[e];
        x[e] = l > 0.f ? __fsub_ru(c, eps) : (l < 0.f ? __fadd_rd(c, eps) : c);
    }
}

// Per-subdomain ascent states (slopes or split multipliers) between a batch, in the alpha_out layout (per ReLU
// layer q a block [n, R, n_q] at n R gbase_q), and a pool of slots ([R, sum_n] each, layer q at R gbase_q).
// Gather: batch <- pool[slot[i]], or -1 (no start) where slot[i] < 0. Scatter: pool[slot[i]] <- batch where
// slot[i] >= 0.
__global__ void bab_state_k(float* __restrict__ pool, const int* __restrict__ slot, int n, int R, long long sum_n,
                            const int* __restrict__ meta_n, const int* __restrict__ meta_g, int nl,
                            float* __restrict__ batch, int scatter) {
    for (int q = 0; q < nl; ++q) {
        const long long nq = meta_n[q], gq = meta_g[q];
        const long long per = (long long)R * nq;
        const long long total = (long long)n * per;
        for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
             e += (long long)gridDim.x * blockDim.x) {
            const long long i = e / per, w = e - i * per;
            const int sl = slot[i];
            float* b = batch + (long long)n * R * gq + e;
            float* pp = pool + (long long)(sl < 0 ? 0 : sl) * R * sum_n + (long long)R * gq + w;
            if (scatter) {
                if (sl >= 0) *pp = *b;
            } else {
                *b = sl >= 0 ? *pp : -1.f;
            }
        }
    }
}

}  // namespace

cudaError_t launch_bab_state(float* pool, const int* slot, int n, int R, long long sum_n, const int* meta_n,
                             const int* meta_g, int nl, float* batch, int scatter, cudaStream_t s) {
    if (n <= 0 || nl <= 0) return cudaSuccess;
    long long g = ((long long)n * R * sum_n + 255) / 256;
    if (g > 148LL * 16) g = 148LL * 16;
    bab_state_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(pool, slot, n, R, sum_n, meta_n, meta_g, nl, batch, scatter);
    return cudaGetLastError();
}

cudaError_t launch_minimiser_points(const float* centre, const float* lam, float eps, long long n, int R, float* x,
                                    cudaStream_t s) {
    long long g = (n * R + 255) / 256;
    if (g > 148LL * 32) g = 148LL * 32;
    minimiser_points_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(centre, lam, eps, n, R, x);
    return cudaGetLastError();
}

cudaError_t launch_bab_pick(const float* pre_lb, const float* pre_ub, int D, const long long* blk_off, const int* blk_n,
                            const int* gbase, int nl, const float* lb_a, const float* lb_b, int R, BabPick* out,
                            cudaStream_t s) {
    if (D <= 0) return cudaSuccess;
    bab_pick_k<<<D, 256, 0, s>>>(pre_lb, pre_ub, D, blk_off, blk_n, gbase, nl, lb_a, lb_b, R, out);
    return cudaGetLastError();
}

cudaError_t launch_repeat_row(const float* src, long long n, int D, float* dst, cudaStream_t s) {
    long long g = (n * D + 255) / 256;
    if (g > 148LL * 32) g = 148LL * 32;
    repeat_row_k<<<(unsigned)(g < 1 ? 1 : g), 256, 0, s>>>(src, n, D, dst);
    return cudaGetLastError();
}

}  // namespace vf
