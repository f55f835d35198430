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
#include "vf_internal.cuh"

namespace vf {

namespace {

constexpr int BK = 8;

template <int BM, int BN>
__global__ void __launch_bounds__(BM * BN / 64)
dense_back_ffma(RowRef A, Relax rx, const float* __restrict__ W, const float* __restrict__ bias, long long M, int K,
                int N, PassGeom pg, int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cst,
                const float* __restrict__ centres, float eps, float* __restrict__ part) {
    constexpr int NT = BM * BN / 64;
    constexpr int TX = BN / 8;
    constexpr int A_ROW_STEP = NT / BK;
    constexpr int A_PER = BM / A_ROW_STEP;
    constexpr int B_PER = BK * BN / NT;
    static_assert(NT % BK == 0 && BM % A_ROW_STEP == 0 && (BK * BN) % NT == 0, "tile shape");
    static_assert(TX <= 32 && (32 % TX) == 0, "row group must sit inside a warp");

    __shared__ __align__(16) float As[2][BK][BM + 4];
    __shared__ __align__(16) float Bs[2][BK][BN + 4];

    const int tid = threadIdx.x;
    const int tx = tid % TX, ty = tid / TX;
    const long long m_base = (long long)blockIdx.x * BM;
    const int n_base = blockIdx.y * BN;
    const bool do_cst = (cst != nullptr) && blockIdx.y == 0;

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
            if (a_ptr[i] != nullptr && k < K) {
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
            b_reg[j] = (kr < K && n < N) ? W[(long long)kr * N + n] : 0.f;
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

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    load_tile(0);
    store_tile(0);
    __syncthreads();
    int cur = 0;
    for (int k0 = 0; k0 < K; k0 += BK) {
        const bool more = (k0 + BK) < K;
        if (more) load_tile(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][BM / 2 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][BN / 2 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (more) store_tile(cur ^ 1);
        __syncthreads();
        cur ^= 1;
    }

    // Row constants: the BK threads that loaded a row's columns hold its partial sums.
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
        for (int i = 0; i < 8; ++i) {
            const long long m = m_base + ((i < 4) ? ty * 4 + i : BM / 2 + ty * 4 + (i - 4));
            float s = 0.f;
            if (m < M) {
                const float* c = centres + ((pg.pass_m0 + m) / pg.R_pass) * (long long)N;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int n = n_base + ((j < 4) ? tx * 4 + j : BN / 2 + tx * 4 + (j - 4));
                    if (n < N) s += fmaf(acc[i][j], c[n], -eps * fabsf(acc[i][j]));
                }
            }
#pragma unroll
            for (int off = TX / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (tx == 0 && m < M) part[(long long)blockIdx.y * M + m] = s;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const long long m = m_base + ((i < 4) ? ty * 4 + i : BM / 2 + ty * 4 + (i - 4));
            if (m >= M) continue;
            float* o = out + m * ld_out;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = n_base + ((j < 4) ? tx * 4 + j : BN / 2 + tx * 4 + (j - 4));
                if (n < N) o[n] = (out_mode == OUT_ACCUM ? o[n] : 0.f) + acc[i][j];
            }
        }
    }
}

}  // namespace

int dense_back_tiles_n(int N) { return N <= 64 ? (N + 63) / 64 : (N + 127) / 128; }

cudaError_t launch_dense_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M, int K, int N,
                              PassGeom pg, int out_mode, float* out, long long ld_out, float* cst,
                              const float* centres, float eps, float* part, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    if (N <= 64) {
        dim3 grid((unsigned)((M + 63) / 64), (unsigned)((N + 63) / 64));
        dense_back_ffma<64, 64><<<grid, 64, 0, s>>>(A, rx, W, bias, M, K, N, pg, out_mode, out, ld_out, cst, centres,
                                                    eps, part);
    } else {
        dim3 grid((unsigned)((M + 127) / 128), (unsigned)((N + 127) / 128));
        dense_back_ffma<128, 128><<<grid, 256, 0, s>>>(A, rx, W, bias, M, K, N, pg, out_mode, out, ld_out, cst,
                                                       centres, eps, part);
    }
    return cudaGetLastError();
}

}  // namespace vf
