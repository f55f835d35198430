// CROWN back-substitution through a dense node on the 5th-generation tensor cores (sm_100a):
// tcgen05.mma kind::tf32 with the 3xTF32 split, operands staged by TMA, accumulator in TMEM.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (the linear relaxation matrices A that CROWN carries back
// through every layer) and §2.1 (ReLU relaxation slopes fixed by intermediate bounds).
//
// Computes, for one row block of M rows (same contract as the FFMA kernel in k_back.cu):
//   x      = A[m, k]  (coefficients over a ReLU output, or over the node output)
//   r      = relax(x) = x >= 0 ? x * lo[b, k] : x * up[b, k]        (identity if no relaxation)
//   cst[m] += sum_k min(x, 0) * t[b, k] + r * bias[k]
//   out[m, n] (=, +=) sum_k r * W[k, n]      or, concretised, part[tile, m] = sum_n v c_b[n] - eps |v|
//
// 3xTF32 (error-compensated split, Ootomo & Yokota 2022): r = r_hi + r_lo with r_hi = r truncated
// to tf32 (10 mantissa bits, exact in fp32) and r_lo = r - r_hi; the same for W, split once at
// network creation. Three MMAs accumulate r_hi W_hi + r_hi W_lo + r_lo W_hi in fp32, which
// leaves an error near 2^-21 relative per product instead of tf32's 2^-11.
//
// Roles in a CTA of 6 warps (one 128-row x BN-column output tile):
//   warp 0: TMA producer (raw A tile, W_hi and W_lo tiles) and TMEM allocator;
//   warp 1: one thread issues the MMAs and commits them to mbarriers;
//   warps 2-5: one thread per row -- relax + split A into the swizzled smem operand layout, keep
//              the row constant, then read the accumulator from TMEM and write the epilogue.
// All waits are bounded: on expiry a shared abort flag stops every role, the producer waits (also
// bounded) for its copies in flight, TMEM is freed and the kernel reports through *err.
#include <cuda.h>

#include "vf_internal.cuh"
#include "vf_tc.cuh"

namespace vf {

namespace {

constexpr int BM = 128;
constexpr int BK = 32;                 // one 128-byte swizzle row of fp32
constexpr int TILE_A = BM * BK * 4;    // 16 KB
constexpr int MAX_BN = 256;
constexpr int NUM_THREADS = 192;
constexpr long long WAIT_CYCLES = 4000000000LL;  // ~2 s at boost clock

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait; returns false (and raises the CTA abort flag) when it gives up or sees abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const long long t0 = clock64();
    while (!mbar_test(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_CYCLES) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint32_t idesc_tf32(int n) {
    // D fp32, A/B tf32, both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

struct TcParams {
    long long M;
    int K, N, BN, n_stages, ntiles_n;
    int a_row_mode;        // 0: local rows y = m; 1: shared block y = (m0 + m) % RA
    long long a_m0, a_RA;  // for mode 1
    PassGeom pg;
    int out_mode;
    float* out;
    long long ld_out;
    float* cst;
    const float* centres;
    float eps;
    float* part;
    const float* bias;
    Relax rx;
    int* err;
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
dense_back_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBhi,
              const __grid_constant__ CUtensorMap tmBlo, TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned carve-up: per stage [A (raw, then hi in place) | A_lo | B_hi | B_lo]
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bbytes = p.BN * BK * 4;
    const int stage_bytes = 2 * TILE_A + 2 * bbytes;
    __shared__ uint64_t full_bar[4], xform_bar[4], empty_bar[4], acc_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.n_stages;
    const int nk = (p.K + BK - 1) / BK;
    const long long m_tile = blockIdx.x;
    const int n_tile = blockIdx.y;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&xform_bar[s], 128);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int* abort_flag = &abort_sh;

    if (warp == 0) {
        if (lane == 0) {
            const int ya = (p.a_row_mode == 0) ? (int)(m_tile * BM) : (int)((p.a_m0 + m_tile * BM) % p.a_RA);
            const int yb = n_tile * p.BN;
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % S;
                if (kb >= S && !mbar_wait(&empty_bar[s], ((kb / S) - 1) & 1, abort_flag)) break;
                uint8_t* st = base + (size_t)s * stage_bytes;
                mbar_expect_tx(&full_bar[s], TILE_A + 2 * bbytes);
                tma_load_2d(st, &tmA, &full_bar[s], kb * BK, ya);
                tma_load_2d(st + 2 * TILE_A, &tmBhi, &full_bar[s], kb * BK, yb);
                tma_load_2d(st + 2 * TILE_A + bbytes, &tmBlo, &full_bar[s], kb * BK, yb);
                issued = kb + 1;
            }
            if (*abort_flag) {
                // drain: wait (bounded) for every copy this thread issued that nobody consumed
                for (int kb = (issued > S ? issued - S : 0); kb < issued; ++kb) {
                    const long long t0 = clock64();
                    while (!mbar_test(&full_bar[kb % S], (kb / S) & 1) && clock64() - t0 < WAIT_CYCLES) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_tf32(p.BN);
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (kb / S) & 1;
                if (!mbar_wait(&xform_bar[s], ph, abort_flag)) break;
                if (!mbar_wait(&full_bar[s], ph, abort_flag)) break;
                tc_fence_after();
                uint8_t* st = base + (size_t)s * stage_bytes;
                const uint64_t da_hi = sw128_desc(smem_u32(st));
                const uint64_t da_lo = sw128_desc(smem_u32(st + TILE_A));
                const uint64_t db_hi = sw128_desc(smem_u32(st + 2 * TILE_A));
                const uint64_t db_lo = sw128_desc(smem_u32(st + 2 * TILE_A + bbytes));
#pragma unroll
                for (int kk = 0; kk < BK / 8; ++kk) {
                    const uint64_t off = (uint64_t)(kk * 32) >> 4;  // 8 tf32 = 32 bytes along K
                    const uint32_t first = (kb > 0 || kk > 0) ? 1u : 0u;
                    mma_tf32(tmem, da_lo + off, db_hi + off, idesc, first);
                    mma_tf32(tmem, da_hi + off, db_lo + off, idesc, 1u);
                    mma_tf32(tmem, da_hi + off, db_hi + off, idesc, 1u);
                }
                mma_commit(&empty_bar[s]);
            }
            mma_commit(&acc_bar);
            // never free TMEM under MMAs still in flight, even after an abort
            const long long t0 = clock64();
            while (!mbar_test(&acc_bar, 0) && clock64() - t0 < WAIT_CYCLES) {
            }
        }
    } else {
        // ------------------------------------------------------------ transform + epilogue
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;           // row of the tile owned by this thread
        const long long m = m_tile * BM + row;
        const bool valid = m < p.M;
        const long long b = (p.pg.pass_m0 + m) / p.pg.R_pass;
        const bool do_cst = (p.cst != nullptr) && n_tile == 0;
        float cacc = 0.f;
        const float4* P = p.rx.P;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % S;
            if (!mbar_wait(&full_bar[s], (kb / S) & 1, abort_flag)) break;
            uint8_t* st = base + (size_t)s * stage_bytes;
            float4* arow = reinterpret_cast<float4*>(st + row * 128);
            float4* lrow = reinterpret_cast<float4*>(st + TILE_A + row * 128);
            const int k0 = kb * BK;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int pc = c ^ (row & 7);  // 128-byte swizzle: chunk c of this row sits at pc
                float4 x = arow[pc];
                float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = k0 + c * 4 + j;
                    float r = v[j];
                    if (P != nullptr && valid && k < p.K) {
                        const float4 pr = __ldg(&P[b * p.K + k]);
                        r = (v[j] >= 0.f) ? v[j] * pr.x : v[j] * pr.y;
                        if (p.rx.count_const) cacc = fmaf(fminf(v[j], 0.f), pr.z, cacc);
                    }
                    if (do_cst && p.bias != nullptr && valid && k < p.K) cacc = fmaf(r, __ldg(&p.bias[k]), cacc);
                    v[j] = r;
                }
                const float4 hi = make_float4(tf32_hi(v[0]), tf32_hi(v[1]), tf32_hi(v[2]), tf32_hi(v[3]));
                arow[pc] = hi;
                lrow[pc] = make_float4(v[0] - hi.x, v[1] - hi.y, v[2] - hi.z, v[3] - hi.w);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&xform_bar[s]);
        }
        if (do_cst && valid && !*abort_flag) p.cst[m] += cacc;

        // epilogue: accumulator rows from TMEM
        const bool acc_ready = __all_sync(0xffffffffu, mbar_wait(&acc_bar, 0, abort_flag));
        if (acc_ready) {
            tc_fence_after();
            const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
            const int n0 = n_tile * p.BN;
            float conc = 0.f;
            const float* crow = (p.out_mode == OUT_CONCRETIZE && valid) ? p.centres + b * (long long)p.N : nullptr;
            float* orow = (p.out_mode != OUT_CONCRETIZE && valid) ? p.out + m * p.ld_out : nullptr;
            for (int c0 = 0; c0 < p.BN; c0 += 32) {
                float v[32];
                tmem_ld32(lane_addr + c0, v);
                if (!valid) continue;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int n = n0 + c0 + j;
                    if (c0 + j >= p.BN || n >= p.N) break;
                    if (crow != nullptr) {
                        conc += fmaf(v[j], __ldg(&crow[n]), -p.eps * fabsf(v[j]));
                    } else {
                        orow[n] = (p.out_mode == OUT_ACCUM ? orow[n] : 0.f) + v[j];
                    }
                }
            }
            if (p.out_mode == OUT_CONCRETIZE && valid) p.part[(long long)n_tile * p.M + m] = conc;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256) : "memory");
    }
    if (threadIdx.x == 0 && abort_sh && p.err != nullptr) atomicExch(p.err, 1);
}

// ---------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D fp32 tensor map: inner dimension `cols` (contiguous), `rows` rows `ld` elements apart,
// box of 32 x box_rows, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const float* ptr, long long cols, long long rows, long long ld, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 4)};
    cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int pick_bn(int N, int* ntiles) {
    int t = (N + MAX_BN - 1) / MAX_BN;
    int bn = (N + t - 1) / t;
    bn = (bn + 15) / 16 * 16;
    *ntiles = (N + bn - 1) / bn;
    return bn;
}

}  // namespace

int dense_back_tc_tiles_n(int N) {
    int t;
    pick_bn(N, &t);
    return t;
}

bool dense_back_tc_supported(const RowRef& A, long long M, int K, int N, PassGeom pg) {
    if (K % 4 != 0 || K < 32 || N < 16) return false;
    if ((reinterpret_cast<uintptr_t>(A.ptr) & 15) != 0 || (A.ld % 4) != 0) return false;
    if (A.RA == kHugeRows && A.sB == 0 && A.m0 == 0) return M < (1LL << 31);  // chunk-local rows
    if (A.sB == 0 && A.RA % BM == 0 && A.m0 % BM == 0) return true;            // one block shared by all centres
    (void)pg;
    return false;
}

cudaError_t launch_dense_back_tc(const RowRef& A, Relax rx, const float* Wt_hi, const float* Wt_lo, const float* bias,
                                 long long M, int K, int N, PassGeom pg, int out_mode, float* out, long long ld_out,
                                 float* cst, const float* centres, float eps, float* part, int* err, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    TcParams p{};
    p.M = M;
    p.K = K;
    p.N = N;
    p.BN = pick_bn(N, &p.ntiles_n);
    const int stage_bytes = 2 * TILE_A + 2 * p.BN * BK * 4;
    p.n_stages = stage_bytes * 4 + 1024 <= 220 * 1024 ? 4 : (stage_bytes * 3 + 1024 <= 220 * 1024 ? 3 : 2);
    const size_t smem = (size_t)stage_bytes * p.n_stages + 1024;
    CUtensorMap ta, tbh, tbl;
    long long a_rows;
    if (A.RA == kHugeRows) {
        p.a_row_mode = 0;
        a_rows = M;
    } else {
        p.a_row_mode = 1;
        p.a_m0 = A.m0;
        p.a_RA = A.RA;
        a_rows = A.RA;
    }
    if (!make_map(&ta, A.ptr, K, a_rows, A.ld, BM) || !make_map(&tbh, Wt_hi, K, N, K, p.BN) ||
        !make_map(&tbl, Wt_lo, K, N, K, p.BN))
        return cudaErrorInvalidValue;
    p.pg = pg;
    p.out_mode = out_mode;
    p.out = out;
    p.ld_out = ld_out;
    p.cst = cst;
    p.centres = centres;
    p.eps = eps;
    p.part = part;
    p.bias = bias;
    p.rx = rx;
    p.err = err;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(dense_back_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    dim3 grid((unsigned)((M + BM - 1) / BM), (unsigned)p.ntiles_n);
    dense_back_tc<<<grid, NUM_THREADS, smem, s>>>(ta, tbh, tbl, p);
    return cudaGetLastError();
}

}  // namespace vf
