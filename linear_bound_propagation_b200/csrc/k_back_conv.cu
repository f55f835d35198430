// CROWN back-substitution through a convolution node (transposed convolution of the rows).
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.2 and §4.2 (bounds through convolutional layers) and §1
// (the linear relaxation matrices A).
//
// For z = conv(h) + b and coefficient rows Lambda over z (length C_out * H_out * W_out):
//   Lambda_h[ci, y, x] = sum_{co, p, q} Lambda[co, (y + pad - p) / s, (x + pad - q) / s] * W[co, ci, p, q]
//   (terms whose source index is fractional or outside the output map are absent)
//   const += sum_{co, i, j} Lambda[co, i, j] * b[co]
// Relaxation of a ReLU output is applied as each row is staged in shared memory. One CTA
// owns a whole row at a time (persistent over rows, the weights staged once), so the row
// constant and, for the node that reads the input, the concretisation reduce inside the CTA
// in a fixed order.
#include "vf_internal.cuh"

namespace vf {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0)
        for (int i = 0; i < kThreads / 32; ++i) t += red[i];
    __syncthreads();
    return t;  // valid in thread 0
}

__global__ void __launch_bounds__(kThreads)
conv_back_ffma(RowRef A, Relax rx, const float* __restrict__ W, const float* __restrict__ bias, long long M, ConvGeom g,
               PassGeom pg, int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cst,
               const float* __restrict__ centres, float eps) {
    extern __shared__ float4 smem4[];
    __shared__ float red[kThreads / 32];
    float* smem = reinterpret_cast<float*>(smem4);
    const int ci4 = (g.ci + 3) / 4 * 4;
    const int kk = g.k * g.k;
    const int nW = g.co * kk * ci4;
    float* Ws = smem;        // [co][p][q][ci4]
    float* Ls = smem + nW;   // [co][i][j] relaxed row
    const int hw_o = g.ho * g.wo;
    const int nOut = g.co * hw_o;
    const int S = g.h * g.w;
    const long long nIn = (long long)g.ci * S;
    const int tid = threadIdx.x;

    for (int e = tid; e < nW; e += kThreads) {
        const int ci = e % ci4;
        int rest = e / ci4;
        const int q = rest % g.k;
        rest /= g.k;
        const int p = rest % g.k;
        const int co = rest / g.k;
        Ws[e] = (ci < g.ci) ? W[(((long long)co * g.ci + ci) * g.k + p) * g.k + q] : 0.f;
    }
    __syncthreads();

    const int items = (ci4 / 4) * S;
    const int wstride = kk * ci4;  // floats between consecutive co in Ws
    for (long long m = blockIdx.x; m < M; m += gridDim.x) {
        const float* arow = A.row(m);
        const long long b = (pg.pass_m0 + m) / pg.R_pass;
        float cs = 0.f;
        for (int j = tid; j < nOut; j += kThreads) {
            const float x = arow[j];
            float r = x;
            if (rx.P != nullptr) {
                const float4 pr = rx.P[b * nOut + j];
                r = (x >= 0.f) ? x * pr.x : x * pr.y;
                if (rx.count_const) cs = fmaf(fminf(x, 0.f), pr.z, cs);
            }
            if (bias != nullptr) cs = fmaf(r, bias[j / hw_o], cs);
            Ls[j] = r;
        }
        __syncthreads();
        float conc = 0.f;
        for (int it = tid; it < items; it += kThreads) {
            const int cg = it / S, sp = it % S;
            const int y = sp / g.w, x = sp % g.w;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            for (int p = 0; p < g.k; ++p) {
                const int ty = y + g.pad - p;
                if (ty < 0 || (ty % g.stride) != 0) continue;
                const int oi = ty / g.stride;
                if (oi >= g.ho) continue;
                for (int q = 0; q < g.k; ++q) {
                    const int tx = x + g.pad - q;
                    if (tx < 0 || (tx % g.stride) != 0) continue;
                    const int oj = tx / g.stride;
                    if (oj >= g.wo) continue;
                    const float* lp = Ls + oi * g.wo + oj;
                    const float* wp = Ws + (p * g.k + q) * ci4 + cg * 4;
                    for (int co = 0; co < g.co; ++co) {
                        const float lam = lp[co * hw_o];
                        const float4 w4 = *reinterpret_cast<const float4*>(wp + co * wstride);
                        a0 = fmaf(lam, w4.x, a0);
                        a1 = fmaf(lam, w4.y, a1);
                        a2 = fmaf(lam, w4.z, a2);
                        a3 = fmaf(lam, w4.w, a3);
                    }
                }
            }
            const float av[4] = {a0, a1, a2, a3};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int ci = cg * 4 + t;
                if (ci >= g.ci) break;
                const long long idx = (long long)ci * S + sp;
                if (out_mode == OUT_CONCRETIZE) {
                    conc += fmaf(av[t], centres[b * nIn + idx], -eps * fabsf(av[t]));
                } else {
                    float* o = out + m * ld_out + idx;
                    *o = (out_mode == OUT_ACCUM ? *o : 0.f) + av[t];
                }
            }
        }
        const float tot = block_sum(cs + conc, red);
        if (tid == 0 && cst != nullptr) cst[m] += tot;
        // block_sum ends with a barrier, so Ls may be overwritten by the next row.
    }
}

}  // namespace

size_t conv_back_smem_bytes(const ConvGeom& g) {
    const size_t ci4 = (size_t)(g.ci + 3) / 4 * 4;
    return ((size_t)g.co * g.k * g.k * ci4 + (size_t)g.co * g.ho * g.wo) * sizeof(float);
}

cudaError_t launch_conv_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M,
                             const ConvGeom& g, PassGeom pg, int out_mode, float* out, long long ld_out, float* cst,
                             const float* centres, float eps, int num_sms, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    const size_t smem = conv_back_smem_bytes(g);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(conv_back_ffma, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv_back_ffma, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    long long grid = (long long)num_sms * per_sm;
    if (grid > M) grid = M;
    conv_back_ffma<<<(unsigned)grid, kThreads, smem, s>>>(A, rx, W, bias, M, g, pg, out_mode, out, ld_out, cst,
                                                          centres, eps);
    return cudaGetLastError();
}

}  // namespace vf
