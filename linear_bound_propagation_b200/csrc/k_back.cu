// CROWN back-substitution through a dense node, as one tiled fp32 FFMA contraction.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (the linear relaxation matrices A that CROWN carries
// backwards) and §2.1 (the ReLU relaxation slopes fixed by intermediate bounds).
//
// For a dense node z = W h + b and coefficient rows Lambda over z:
//   const[m]  += sum_k Lambda[m, k] * b[k]             (bias term)
//   Lambda_h   = Lambda . W                            (M x K) . (K x N)
// When the rows arrive over a ReLU output, the relaxation is applied as A is loaded:
//   x >= 0 -> x * lo,  x < 0 -> x * up,  const += min(x, 0) * t
// The epilogue either stores Lambda_h, adds it into an existing buffer, or -- for the node
// that reads the input box -- concretises it at once (Lambda_h . c - eps * |Lambda_h|),
// writing one partial per N tile that a later pass sums in a fixed order.
#include <cooperative_groups.h>

#include "vf_internal.cuh"

namespace cg = cooperative_groups;

namespace vf {

namespace {

constexpr int BK = 8;

// Each thread owns a TM x TM block of outputs (TM = 8: two 4-row and two 4-column halves, TM = 4: one
// 4 x 4 block). SPLIT: the launch is a cluster of gridDim.z CTAs over the same output tile, CTA rank r
// taking the r-th slice of the K loop. The ranks park their partial tiles (and row-constant partials)
// in shared memory and, after a cluster barrier, each rank sums an equal share of the tile's rows over
// the cluster's distributed shared memory in rank order, so a result does not depend on scheduling.
// A dot product of K terms is still one sum of those K products (in a different association), so the
// sound mode's per-product rounding bound gamma_K covers it unchanged.
template <int BM, int BN, int TM, bool SPLIT>
__global__ void __launch_bounds__(BM * BN / (TM * TM))
dense_back_ffma(RowRef A, Relax rx, const float* __restrict__ W, const float* __restrict__ bias, long long M, int K,
                int N, PassGeom pg, int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cst,
                const float* __restrict__ centres, float eps, float* __restrict__ part) {
    constexpr int NT = BM * BN / (TM * TM);
    constexpr int TX = BN / TM;
    constexpr int A_ROW_STEP = NT / BK;
    constexpr int A_PER = BM / A_ROW_STEP;
    constexpr int B_PER = BK * BN / NT;
    static_assert(TM == 4 || TM == 8, "thread tile");
    static_assert(NT % BK == 0 && BM % A_ROW_STEP == 0 && (BK * BN) % NT == 0, "tile shape");
    static_assert(TX <= 32 && (32 % TX) == 0, "row group must sit inside a warp");
    static_assert(!SPLIT || (NT % 32 == 0 && BN % 32 == 0), "split epilogue: whole warps over 32-column groups");

    __shared__ __align__(16) float As[2][BK][BM + 4];
    __shared__ __align__(16) float Bs[2][BK][BN + 4];

    const int tid = threadIdx.x;
    const int tx = tid % TX, ty = tid / TX;
    const long long m_base = (long long)blockIdx.x * BM;
    const int n_base = blockIdx.y * BN;
    const bool do_cst = (cst != nullptr) && blockIdx.y == 0;

    // K range of this CTA: all of it, or the rank's share of the BK-wide slices
    int k_begin = 0, k_end = K;
    if constexpr (SPLIT) {
        const int ks = (int)gridDim.z, r = (int)blockIdx.z;
        const int nk = (K + BK - 1) / BK;
        k_begin = (int)((long long)r * nk / ks) * BK;
        k_end = min(K, (int)((long long)(r + 1) * nk / ks) * BK);
    }

    const int a_col = tid % BK;
    const int a_row0 = tid / BK;
    const float* a_ptr[A_PER];
    long long a_cb[A_PER];
    float cst_acc[A_PER];
#pragma unroll
    for (int i = 0; i < A_PER; ++i) {
        long long m = m_base + a_row0 + i * A_ROW_STEP;
        a_ptr[i] = (m < M) ? A.row(m) : nullptr;
        a_cb[i] = (pg.pass_m0 + m) / pg.R_pass;
        cst_acc[i] = 0.f;
    }

    float a_reg[A_PER], b_reg[B_PER];
    auto load_tile = [&](int k0) {
        const int k = k0 + a_col;
#pragma unroll
        for (int i = 0; i < A_PER; ++i) {
            float x = 0.f;
            if (a_ptr[i] != nullptr && k < k_end) {
                x = a_ptr[i][k];
                float r = x;
                if (rx.P != nullptr) {
                    const float4 p = rx.P[a_cb[i] * K + k];
                    r = (x >= 0.f) ? x * p.x : x * p.y;
                    if (do_cst && rx.count_const) cst_acc[i] = fmaf(fminf(x, 0.f), p.z, cst_acc[i]);
                }
                if (do_cst && bias != nullptr) cst_acc[i] = fmaf(r, bias[k], cst_acc[i]);
                x = r;
            }
            a_reg[i] = x;
        }
#pragma unroll
        for (int j = 0; j < B_PER; ++j) {
            const int e = tid + j * NT;
            const int kk = e / BN, nn = e % BN;
            const int kr = k0 + kk, n = n_base + nn;
            b_reg[j] = (kr < k_end && n < N) ? W[(long long)kr * N + n] : 0.f;
        }
    };
    auto store_tile = [&](int buf) {
#pragma unroll
        for (int i = 0; i < A_PER; ++i) As[buf][a_col][a_row0 + i * A_ROW_STEP] = a_reg[i];
#pragma unroll
        for (int j = 0; j < B_PER; ++j) {
            const int e = tid + j * NT;
            Bs[buf][e / BN][e % BN] = b_reg[j];
        }
    };

    float acc[TM][TM];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) acc[i][j] = 0.f;

    load_tile(k_begin);
    store_tile(0);
    __syncthreads();
    int cur = 0;
    for (int k0 = k_begin; k0 < k_end; k0 += BK) {
        const bool more = (k0 + BK) < k_end;
        if (more) load_tile(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[TM], b[TM];
            const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
            a[0] = a0.x, a[1] = a0.y, a[2] = a0.z, a[3] = a0.w;
            b[0] = b0.x, b[1] = b0.y, b[2] = b0.z, b[3] = b0.w;
            if constexpr (TM == 8) {
                const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][BM / 2 + ty * 4]);
                const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][BN / 2 + tx * 4]);
                a[4] = a1.x, a[5] = a1.y, a[6] = a1.z, a[7] = a1.w;
                b[4] = b1.x, b[5] = b1.y, b[6] = b1.z, b[7] = b1.w;
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TM; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (more) store_tile(cur ^ 1);
        __syncthreads();
        cur ^= 1;
    }
    // tile-local row and column of the thread's output (i, j)
    auto row_of = [&](int i) { return (i < 4) ? ty * 4 + i : BM / 2 + ty * 4 + (i - 4); };
    auto col_of = [&](int j) { return (j < 4) ? tx * 4 + j : BN / 2 + tx * 4 + (j - 4); };

    // Row constants: the BK threads that loaded a row's columns hold its partial sums.
    if constexpr (SPLIT) {
        __shared__ __align__(16) float Cs[BM][BN + 4];
        __shared__ float Ccst[BM];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TM; ++j) Cs[row_of(i)][col_of(j)] = acc[i][j];
        if (do_cst) {
#pragma unroll
            for (int i = 0; i < A_PER; ++i) {
                float v = cst_acc[i];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                if (a_col == 0) Ccst[a_row0 + i * A_ROW_STEP] = v;
            }
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int ks = (int)gridDim.z, r = (int)blockIdx.z;
        const int rows_per = BM / ks;  // ks divides BM (the launcher picks a power of two)
        const int warp = tid / 32, lane = tid % 32;
        for (int rr = warp; rr < rows_per; rr += NT / 32) {
            const int row = r * rows_per + rr;
            const long long m = m_base + row;
            if (m >= M) break;
            float v[BN / 32];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) v[c] = 0.f;
            float cv = 0.f;
            for (int q = 0; q < ks; ++q) {  // rank order: the same sum on every run
                const float* cq = cluster.map_shared_rank(&Cs[0][0], q) + row * (BN + 4);
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) v[c] += cq[lane + 32 * c];
                if (do_cst && lane == 0) cv += cluster.map_shared_rank(Ccst, q)[row];
            }
            if (do_cst && lane == 0) cst[m] += cv;
            if (out_mode == OUT_CONCRETIZE) {
                const float* c = centres + ((pg.pass_m0 + m) / pg.R_pass) * (long long)N;
                float sum = 0.f;
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) {
                    const int n = n_base + lane + 32 * cc;
                    if (n < N) sum += fmaf(v[cc], c[n], -eps * fabsf(v[cc]));
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane == 0) part[(long long)blockIdx.y * M + m] = sum;
            } else {
                float* o = out + m * ld_out;
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) {
                    const int n = n_base + lane + 32 * cc;
                    if (n < N) o[n] = (out_mode == OUT_ACCUM ? o[n] : 0.f) + v[cc];
                }
            }
        }
        cluster.sync();  // every rank's tile stays in shared memory until the others have read it
        return;
    }

    if (do_cst) {
#pragma unroll
        for (int i = 0; i < A_PER; ++i) {
            float v = cst_acc[i];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            const long long m = m_base + a_row0 + i * A_ROW_STEP;
            if (a_col == 0 && m < M) cst[m] += v;
        }
    }

    if (out_mode == OUT_CONCRETIZE) {
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const long long m = m_base + row_of(i);
            float s = 0.f;
            if (m < M) {
                const float* c = centres + ((pg.pass_m0 + m) / pg.R_pass) * (long long)N;
#pragma unroll
                for (int j = 0; j < TM; ++j) {
                    const int n = n_base + col_of(j);
                    if (n < N) s += fmaf(acc[i][j], c[n], -eps * fabsf(acc[i][j]));
                }
            }
#pragma unroll
            for (int off = TX / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (tx == 0 && m < M) part[(long long)blockIdx.y * M + m] = s;
        }
    } else {
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const long long m = m_base + row_of(i);
            if (m >= M) continue;
            float* o = out + m * ld_out;
#pragma unroll
            for (int j = 0; j < TM; ++j) {
                const int n = n_base + col_of(j);
                if (n < N) o[n] = (out_mode == OUT_ACCUM ? o[n] : 0.f) + acc[i][j];
            }
        }
    }
}

// Cluster size for the split-K kernel: doubled while the launch stays within two CTAs per SM, at most 8
// (the portable cluster limit), a power of two (it divides the tile's 32 rows), and at least two BK slices
// per rank.
int split_ways(long long ctas, int K, int num_sms) {
    int ks = 1;
    while (ks < 8 && ctas * ks * 2 <= 2LL * num_sms && (long long)(ks * 2) * 2 * BK <= K) ks *= 2;
    return ks;
}

template <int BN>
cudaError_t launch_split(const RowRef& A, Relax rx, const float* W, const float* bias, long long M, int K, int N,
                         PassGeom pg, int out_mode, float* out, long long ld_out, float* cst, const float* centres,
                         float eps, float* part, int ks, cudaStream_t s) {
    constexpr int BM = 32;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((M + BM - 1) / BM), (unsigned)((N + BN - 1) / BN), (unsigned)ks);
    cfg.blockDim = dim3(BM * BN / 16);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)ks;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, dense_back_ffma<BM, BN, 4, true>, A, rx, W, bias, M, K, N, pg, out_mode, out,
                              ld_out, cst, centres, eps, part);
}

int sm_count() {
    static int n = 0;  // one device per process in practice; the count only steers the tile choice
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                      cudaSuccess && v > 0)
            n = v;
        else
            return 148;
    }
    return n;
}

}  // namespace

int dense_back_tiles_n(int N) { return N <= 64 ? (N + 63) / 64 : (N + 127) / 128; }

// Tile choice. Large launches: 128 x 128 tiles of 8 x 8 outputs per thread (64 x 64 when N <= 64). A
// launch whose large tiles would not fill the SMs (the few rows of a branch-and-bound batch, a small
// network) takes 32-row tiles of 4 x 4 outputs per thread with K split over a cluster. The column tiles
// are the same width either way, so the number of concretisation partials per row does not change.
cudaError_t launch_dense_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M, int K, int N,
                              PassGeom pg, int out_mode, float* out, long long ld_out, float* cst,
                              const float* centres, float eps, float* part, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    const int sms = sm_count();
    const int tn = dense_back_tiles_n(N);
    const long long big_tiles = (N <= 64 ? (M + 63) / 64 : (M + 127) / 128) * (long long)tn;
    if (big_tiles < sms && M < (1LL << 31)) {
        const int ks = split_ways(((M + 31) / 32) * tn, K, sms);
        return N <= 64 ? launch_split<64>(A, rx, W, bias, M, K, N, pg, out_mode, out, ld_out, cst, centres, eps,
                                          part, ks, s)
                       : launch_split<128>(A, rx, W, bias, M, K, N, pg, out_mode, out, ld_out, cst, centres, eps,
                                           part, ks, s);
    }
    if (N <= 64) {
        dim3 grid((unsigned)((M + 63) / 64), (unsigned)((N + 63) / 64));
        dense_back_ffma<64, 64, 8, false><<<grid, 64, 0, s>>>(A, rx, W, bias, M, K, N, pg, out_mode, out, ld_out,
                                                              cst, centres, eps, part);
    } else {
        dim3 grid((unsigned)((M + 127) / 128), (unsigned)((N + 127) / 128));
        dense_back_ffma<128, 128, 8, false><<<grid, 256, 0, s>>>(A, rx, W, bias, M, K, N, pg, out_mode, out,
                                                                 ld_out, cst, centres, eps, part);
    }
    return cudaGetLastError();
}

}  // namespace vf
