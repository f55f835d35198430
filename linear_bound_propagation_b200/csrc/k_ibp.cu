// Interval bound propagation in centre/radius form.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.1 (IBP, the fast and sound but looser bound used in place
// of CROWN intermediate bounds) and §4.2 (IBP bounds reproduced exactly).
//
//   affine:  centre' = W c + b,   radius' = |W| r     (both products in one pass)
//   ReLU:    [max(c - r, 0), max(c + r, 0)] back to centre/radius
//   add:     centres add, radii add
//   splits:  branch-and-bound subdomains fix the sign of some pre-activations (same page, §2.2 and
//            §4.3: beta-CROWN with branch-and-bound); their intervals are clamped to that sign
#include <cooperative_groups.h>

#include "vf_internal.cuh"

namespace cg = cooperative_groups;

namespace vf {

namespace {

// z[m, n] = sum_k h[m, k] * W[n, k]: plane 0 computes the centre (h = centre, W, + bias), plane 1 the
// radius (h = radius, |W|); the plane is blockIdx.z (/ the cluster size with SPLIT) + z0. Tiles of 64
// rows x 64 columns, 256 threads each owning a 4 x 4 block of outputs; per k the thread reads one float4
// of the staged h tile and one of the staged W tile for 16 FMAs. The next 16-wide k-slice is prefetched
// into registers while the current one is used. With rowsum_abs != nullptr the source is the input box
// with radius eps in every coordinate: the radius is eps * sum_k |W[n, k]| without a product.
// SPLIT: a cluster of ks CTAs shares each output tile, rank r taking the r-th share of the k-slices; the
// partial tiles meet in distributed shared memory and each rank sums 64 / ks of the rows in rank order.
template <bool SPLIT>
__global__ void __launch_bounds__(256)
ibp_dense_k(const float* __restrict__ hc, const float* __restrict__ hr, const float* __restrict__ W,
            const float* __restrict__ Wabs, const float* __restrict__ bias, const float* __restrict__ rowsum_abs,
            float eps, int B, int K, int N, float* __restrict__ zc, float* __restrict__ zr, int z0) {
    constexpr int TM = 64, TN = 64, KB = 16, LDA = TM + 4, LDB = TN + 4;
    __shared__ __align__(16) float As[KB][LDA];
    __shared__ __align__(16) float Bs[KB][LDB];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.x * TM, n0 = blockIdx.y * TN;
    const int ks = SPLIT ? (int)cg::this_cluster().num_blocks() : 1;  // the cluster spans (1, 1, ks) CTAs
    const int rank = SPLIT ? (int)blockIdx.z % ks : 0;
    const bool rad = (int)blockIdx.z / ks + z0 == 1;
    if (rad && rowsum_abs != nullptr) {  // the whole cluster leaves here together: no barrier is pending
        if (rank != 0) return;
        for (int e = tid; e < TM * TN; e += 256) {
            const int m = m0 + e / TN, n = n0 + e % TN;
            if (m < B && n < N) zr[(long long)m * N + n] = eps * rowsum_abs[n];
        }
        return;
    }
    const float* h = rad ? hr : hc;
    const float* w = rad ? Wabs : W;
    const int nk = (K + KB - 1) / KB;
    const int k_begin = (int)((long long)rank * nk / ks) * KB;
    const int k_end = min(K, (int)((long long)(rank + 1) * nk / ks) * KB);
    // loader mapping: 64 rows x 16 k per tile = 1024 values, 4 per thread (k fastest for coalescing)
    float a_reg[4], b_reg[4];
    auto load = [&](int k0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i, row = e / KB, kk = e % KB, k = k0 + kk;
            const int m = m0 + row, n = n0 + row;
            a_reg[i] = (m < B && k < k_end) ? h[(long long)m * K + k] : 0.f;
            b_reg[i] = (n < N && k < k_end) ? w[(long long)n * K + k] : 0.f;
        }
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    load(k_begin);
    for (int k0 = k_begin; k0 < k_end; k0 += KB) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i;
            As[e % KB][e / KB] = a_reg[i];
            Bs[e % KB][e / KB] = b_reg[i];
        }
        __syncthreads();
        if (k0 + KB < k_end) load(k0 + KB);
#pragma unroll
        for (int kk = 0; kk < KB; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
            const float4 bb = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    if constexpr (SPLIT) {
        __shared__ __align__(16) float Cs[TM][TN + 4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(&Cs[ty * 4 + i][tx * 4]) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rows_per = TM / ks;  // ks divides 64 (a power of two)
        for (int e = tid; e < rows_per * TN; e += 256) {
            const int row = rank * rows_per + e / TN, col = e % TN;
            const int m = m0 + row, n = n0 + col;
            float v = 0.f;
            for (int q = 0; q < ks; ++q) v += cluster.map_shared_rank(&Cs[0][0], q)[row * (TN + 4) + col];
            if (m < B && n < N) {
                if (rad)
                    zr[(long long)m * N + n] = v;
                else
                    zc[(long long)m * N + n] = v + bias[n];
            }
        }
        cluster.sync();  // every rank's tile stays in shared memory until the others have read it
        return;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= B) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            if (rad)
                zr[(long long)m * N + n] = acc[i][j];
            else
                zc[(long long)m * N + n] = acc[i][j] + bias[n];
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
            const float* xr = hr != nullptr ? hr + (b * g.ci + ci) * (long long)g.h * g.w : nullptr;
            const float* wp = W + ((long long)co * g.ci + ci) * g.k * g.k;
            const float* wa = Wabs + ((long long)co * g.ci + ci) * g.k * g.k;
            for (int p = 0; p < g.k; ++p) {
                const int y = oi * g.stride - g.pad + p;
                if (y < 0 || y >= g.h) continue;
                for (int q = 0; q < g.k; ++q) {
                    const int x = oj * g.stride - g.pad + q;
                    if (x < 0 || x >= g.w) continue;
                    sc = fmaf(wp[p * g.k + q], xc[y * g.w + x], sc);
                    if (xr != nullptr) sr = fmaf(wa[p * g.k + q], xr[y * g.w + x], sr);
                }
            }
        }
        zc[idx] = bias != nullptr ? sc + bias[co] : sc;
        if (zr != nullptr) zr[idx] = sr;
    }
}

// ReLU of an interval. Under split constraints (split != nullptr, one sign per neuron): a neuron split
// to z <= 0 outputs exactly 0; one split to z >= 0 keeps [max(l, 0), max(u, 0)], the plain result.
__global__ void ibp_relu_k(const float* __restrict__ c, const float* __restrict__ r, long long n,
                           const signed char* __restrict__ split, float* __restrict__ oc, float* __restrict__ orad) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        float lo = fmaxf(c[i] - r[i], 0.f);
        float hi = fmaxf(c[i] + r[i], 0.f);
        if (split != nullptr && split[i] < 0) lo = hi = 0.f;
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

// l = c - r, u = c + r; under split constraints a neuron split to z >= 0 takes l = max(l, 0) and one
// split to z <= 0 takes u = min(u, 0) (an empty interval marks a subdomain with no input).
__global__ void bounds_k(const float* __restrict__ c, const float* __restrict__ r, long long n,
                         const signed char* __restrict__ split, float* __restrict__ lb, float* __restrict__ ub,
                         int sound) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        float l = sound ? __fsub_rd(c[i], r[i]) : c[i] - r[i];
        float u = sound ? __fadd_ru(c[i], r[i]) : c[i] + r[i];
        if (split != nullptr) {
            const signed char sg = split[i];
            if (sg > 0) l = fmaxf(l, 0.f);
            if (sg < 0) u = fminf(u, 0.f);
        }
        lb[i] = l;
        ub[i] = u;
    }
}

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

}  // namespace

namespace {

// Forward products z = h . W^T over `planes` planes (centre and/or radius) starting at plane z0. When
// the 64 x 64 tiles would not fill the SMs, K is split over a cluster of up to 8 CTAs per tile (a power
// of two, at least two 16-wide k-slices per rank).
cudaError_t launch_fwd(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                       const float* rowsum_abs, float eps, int B, int K, int N, float* zc, float* zr, int planes, int z0,
                       cudaStream_t s) {
    if (B <= 0) return cudaSuccess;
    static int sms = 0;
    if (sms == 0) {
        int dev = 0, v = 0;
        sms = (cudaGetDevice(&dev) == cudaSuccess &&
               cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
                  ? v
                  : 148;
    }
    const long long tiles = (long long)((B + 63) / 64) * ((N + 63) / 64) * planes;
    int ks = 1;
    while (ks < 8 && tiles * ks * 2 <= 2LL * sms && ks * 2 * 2 * 16 <= K) ks *= 2;
    if (ks == 1) {
        dim3 grid((B + 63) / 64, (N + 63) / 64, planes);
        ibp_dense_k<false><<<grid, 256, 0, s>>>(hc, hr, W, Wabs, bias, rowsum_abs, eps, B, K, N, zc, zr, z0);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((B + 63) / 64), (unsigned)((N + 63) / 64), (unsigned)(planes * ks));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)ks;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ibp_dense_k<true>, hc, hr, W, Wabs, bias, rowsum_abs, eps, B, K, N, zc, zr, z0);
}

}  // namespace

cudaError_t launch_ibp_dense(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                             const float* rowsum_abs, float eps, int B, int K, int N, float* zc, float* zr,
                             cudaStream_t s) {
    return launch_fwd(hc, hr, W, Wabs, bias, rowsum_abs, eps, B, K, N, zc, zr, 2, 0, s);
}

cudaError_t launch_ibp_radius_rowsum(const float* rowsum_abs, float eps, int B, int N, float* zr, cudaStream_t s) {
    dim3 grid((B + 63) / 64, (N + 63) / 64, 1);  // only the radius of a layer fed by the input box
    ibp_dense_k<false><<<grid, 256, 0, s>>>(nullptr, nullptr, nullptr, nullptr, nullptr, rowsum_abs, eps, B, 0, N,
                                            nullptr, zr, 1);
    return cudaGetLastError();
}

cudaError_t launch_abs_rows_times_wt(const float* A, const float* Wabs, int M, int K, int N, float* out, cudaStream_t s) {
    // only the radius product: out = A |W|^T
    return launch_fwd(A, A, Wabs, Wabs, nullptr, nullptr, 0.f, M, K, N, out, out, 1, 1, s);
}

cudaError_t launch_rows_times_wt(const float* A, const float* W, const float* bias, int M, int K, int N, float* out,
                                 cudaStream_t s) {
    // only the centre product: out = A W^T + bias
    return launch_fwd(A, A, W, W, bias, nullptr, 0.f, M, K, N, out, out, 1, 0, s);
}

cudaError_t launch_ibp_conv(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                            int B, const ConvGeom& g, float* zc, float* zr, cudaStream_t s) {
    const long long total = (long long)B * g.co * g.ho * g.wo;
    ibp_conv_k<<<grid_for(total, 256), 256, 0, s>>>(hc, hr, W, Wabs, bias, B, g, zc, zr);
    return cudaGetLastError();
}

cudaError_t launch_ibp_relu(const float* c, const float* r, long long n, float* oc, float* orad, cudaStream_t s,
                            const signed char* split) {
    ibp_relu_k<<<grid_for(n, 256), 256, 0, s>>>(c, r, n, split, oc, orad);
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

cudaError_t launch_bounds_from_cr(const float* c, const float* r, long long n, float* lb, float* ub, cudaStream_t s,
                                  const signed char* split, int sound) {
    bounds_k<<<grid_for(n, 256), 256, 0, s>>>(c, r, n, split, lb, ub, sound);
    return cudaGetLastError();
}

}  // namespace vf
