// Interval bound propagation in centre/radius form.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.1 (IBP, the fast and sound but looser bound used in place
// of CROWN intermediate bounds) and §4.2 (IBP bounds reproduced exactly).
//
//   affine:  centre' = W c + b,   radius' = |W| r     (both products in one pass)
//   ReLU:    [max(c - r, 0), max(c + r, 0)] back to centre/radius
//   add:     centres add, radii add
#include "vf_internal.cuh"

namespace vf {

namespace {

// z[m, n] = sum_k h[m, k] * W[n, k] for centre (W) and radius (|W|) at once; 64x64 tiles.
__global__ void __launch_bounds__(256)
ibp_dense_k(const float* __restrict__ hc, const float* __restrict__ hr, const float* __restrict__ W,
            const float* __restrict__ Wabs, const float* __restrict__ bias, int B, int K, int N, float* __restrict__ zc,
            float* __restrict__ zr) {
    constexpr int T = 64, KB = 16;
    __shared__ float Ac[KB][T + 1], Ar[KB][T + 1], Bw[KB][T + 1], Ba[KB][T + 1];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.x * T, n0 = blockIdx.y * T;
    float ac[4][4], ar[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) ac[i][j] = ar[i][j] = 0.f;
    for (int k0 = 0; k0 < K; k0 += KB) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i;
            const int row = e / KB, kk = e % KB, k = k0 + kk;
            const int m = m0 + row, n = n0 + row;
            const bool mk = (m < B) && (k < K), nk = (n < N) && (k < K);
            Ac[kk][row] = mk ? hc[(long long)m * K + k] : 0.f;
            Ar[kk][row] = mk ? hr[(long long)m * K + k] : 0.f;
            Bw[kk][row] = nk ? W[(long long)n * K + k] : 0.f;
            Ba[kk][row] = nk ? Wabs[(long long)n * K + k] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KB; ++kk) {
            float a_c[4], a_r[4], b_w[4], b_a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a_c[i] = Ac[kk][ty + 16 * i];
                a_r[i] = Ar[kk][ty + 16 * i];
                b_w[i] = Bw[kk][tx + 16 * i];
                b_a[i] = Ba[kk][tx + 16 * i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    ac[i][j] = fmaf(a_c[i], b_w[j], ac[i][j]);
                    ar[i][j] = fmaf(a_r[i], b_a[j], ar[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= B) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n >= N) continue;
            zc[(long long)m * N + n] = ac[i][j] + bias[n];
            zr[(long long)m * N + n] = ar[i][j];
        }
    }
}

__global__ void ibp_conv_k(const float* __restrict__ hc, const float* __restrict__ hr, const float* __restrict__ W,
                           const float* __restrict__ Wabs, const float* __restrict__ bias, int B, ConvGeom g,
                           float* __restrict__ zc, float* __restrict__ zr) {
    const long long total = (long long)B * g.co * g.ho * g.wo;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int oj = (int)(idx % g.wo);
        long long rest = idx / g.wo;
        const int oi = (int)(rest % g.ho);
        rest /= g.ho;
        const int co = (int)(rest % g.co);
        const long long b = rest / g.co;
        float sc = 0.f, sr = 0.f;
        for (int ci = 0; ci < g.ci; ++ci) {
            const float* xc = hc + (b * g.ci + ci) * (long long)g.h * g.w;
            const float* xr = hr + (b * g.ci + ci) * (long long)g.h * g.w;
            const float* wp = W + ((long long)co * g.ci + ci) * g.k * g.k;
            const float* wa = Wabs + ((long long)co * g.ci + ci) * g.k * g.k;
            for (int p = 0; p < g.k; ++p) {
                const int y = oi * g.stride - g.pad + p;
                if (y < 0 || y >= g.h) continue;
                for (int q = 0; q < g.k; ++q) {
                    const int x = oj * g.stride - g.pad + q;
                    if (x < 0 || x >= g.w) continue;
                    sc = fmaf(wp[p * g.k + q], xc[y * g.w + x], sc);
                    sr = fmaf(wa[p * g.k + q], xr[y * g.w + x], sr);
                }
            }
        }
        zc[idx] = sc + bias[co];
        zr[idx] = sr;
    }
}

__global__ void ibp_relu_k(const float* __restrict__ c, const float* __restrict__ r, long long n, float* __restrict__ oc,
                           float* __restrict__ orad) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float lo = fmaxf(c[i] - r[i], 0.f);
        const float hi = fmaxf(c[i] + r[i], 0.f);
        oc[i] = 0.5f * (hi + lo);
        orad[i] = 0.5f * (hi - lo);
    }
}

__global__ void ibp_add_k(const float* __restrict__ c1, const float* __restrict__ r1, const float* __restrict__ c2,
                          const float* __restrict__ r2, long long n, float* __restrict__ oc, float* __restrict__ orad) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        oc[i] = c1[i] + c2[i];
        orad[i] = r1[i] + r2[i];
    }
}

__global__ void fill_k(float* __restrict__ p, long long n, float v) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = v;
}

__global__ void bounds_k(const float* __restrict__ c, const float* __restrict__ r, long long n, float* __restrict__ lb,
                         float* __restrict__ ub) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        lb[i] = c[i] - r[i];
        ub[i] = c[i] + r[i];
    }
}

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_ibp_dense(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                             int B, int K, int N, float* zc, float* zr, cudaStream_t s) {
    dim3 grid((B + 63) / 64, (N + 63) / 64);
    ibp_dense_k<<<grid, 256, 0, s>>>(hc, hr, W, Wabs, bias, B, K, N, zc, zr);
    return cudaGetLastError();
}

cudaError_t launch_ibp_conv(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                            int B, const ConvGeom& g, float* zc, float* zr, cudaStream_t s) {
    const long long total = (long long)B * g.co * g.ho * g.wo;
    ibp_conv_k<<<grid_for(total, 256), 256, 0, s>>>(hc, hr, W, Wabs, bias, B, g, zc, zr);
    return cudaGetLastError();
}

cudaError_t launch_ibp_relu(const float* c, const float* r, long long n, float* oc, float* orad, cudaStream_t s) {
    ibp_relu_k<<<grid_for(n, 256), 256, 0, s>>>(c, r, n, oc, orad);
    return cudaGetLastError();
}

cudaError_t launch_ibp_add(const float* c1, const float* r1, const float* c2, const float* r2, long long n, float* oc,
                           float* orad, cudaStream_t s) {
    ibp_add_k<<<grid_for(n, 256), 256, 0, s>>>(c1, r1, c2, r2, n, oc, orad);
    return cudaGetLastError();
}

cudaError_t launch_fill(float* p, long long n, float v, cudaStream_t s) {
    fill_k<<<grid_for(n, 256), 256, 0, s>>>(p, n, v);
    return cudaGetLastError();
}

cudaError_t launch_bounds_from_cr(const float* c, const float* r, long long n, float* lb, float* ub, cudaStream_t s) {
    bounds_k<<<grid_for(n, 256), 256, 0, s>>>(c, r, n, lb, ub);
    return cudaGetLastError();
}

}  // namespace vf
