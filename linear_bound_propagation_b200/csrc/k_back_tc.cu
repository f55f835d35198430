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
// Roles in a CTA of 11 warps (one CTA per SM, persistent over 128-row x BN-column output tiles, BN <= 256):
//   warp 0:    TMA producer of the raw A tiles (128 x 32 fp32, 128-byte swizzle) together with the
//              relaxation-table slice of the tile's centres, and owner of the TMEM allocation;
//   warp 10:   TMA producer of the W^T head/remainder tiles (BN x 32 each) into a second ring;
//   warp 1:    one thread issues the kind::tf32 MMAs, A read from TMEM and B from shared memory, and
//              commits each k-block to the barriers that release its A and B stages;
//   warps 2-5: one thread per tile row (= TMEM lane): relax the row's 32 coefficients of the k-block,
//              keep the row constant, split into head/remainder and store both into one of four TMEM A
//              stages (64 columns each);
//   warps 6-9: drain the accumulator (TMEM columns 0..BN-1), hand it back to the MMA and write the
//              epilogue: stores staged through shared memory so global stores are coalesced, or the
//              concretisation against the centre into a per-N-tile partial.
// TMEM: 512 columns per CTA. All waits are bounded: on expiry a shared abort
// flag stops every role, the producers wait (also bounded) for their copies in flight, the MMA
// thread for its MMAs, TMEM is freed and the kernel reports through *err.
#include <cuda.h>

#include <algorithm>

#include "vf_internal.cuh"
#include "vf_tc.cuh"
#include "tc_ptx.cuh"

namespace vf {

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 32;                 // one 128-byte swizzle row of fp32
constexpr int TILE_A = BM * BK * 4;    // 16 KB
constexpr int MAX_BN = 256;
constexpr int NUM_THREADS = 352;  // 11 warps, see the role map above the kernel
// s1 += sum_j v_j * c_j and s2 += sum_j |v_j| over the first CNT values of a TMEM chunk, four independent
// partial sums each (columns at or beyond N hold exact zeros in both the accumulator and the staged centres).
template <int CNT>
__device__ __forceinline__ void conc_chunk(const uint32_t (&v)[32], const float* c, float (&s1)[4], float (&s2)[4]) {
#pragma unroll
    for (int j = 0; j < CNT; j += 4) {
        const float4 cc = *reinterpret_cast<const float4*>(c + j);
        const float x0 = __uint_as_float(v[j]), x1 = __uint_as_float(v[j + 1]);
        const float x2 = __uint_as_float(v[j + 2]), x3 = __uint_as_float(v[j + 3]);
        s1[0] = fmaf(x0, cc.x, s1[0]);
        s1[1] = fmaf(x1, cc.y, s1[1]);
        s1[2] = fmaf(x2, cc.z, s1[2]);
        s1[3] = fmaf(x3, cc.w, s1[3]);
        s2[0] += fabsf(x0);
        s2[1] += fabsf(x1);
        s2[2] += fabsf(x2);
        s2[3] += fabsf(x3);
    }
}

constexpr int MAX_STAGES = 6;
constexpr int A_STAGES = 4;          // TMEM stages of the split A operand (64 columns each)
constexpr uint32_t TMEM_COLS = 512;  // accumulator in [0, 256), A stages in [256, 512)

struct TcParams {
    long long M;
    int K, N, BN, ntiles_n;
    long long ntiles;               // (M tiles) x (N tiles); CTA i takes tiles i, i + grid, ...
    int b_stages, r_stages, nbp;    // B ring depth, raw-A ring depth, centres per P box
    int nbw;                        // centres a warp's 32 rows can span (epilogue staging)
    int b_off, r_off, p_off, s_off; // byte offsets of the rings and the epilogue staging
    int s_floats;                   // epilogue staging floats per warp
    int a_row_mode;                 // 0: local rows y = m; 1: shared block y = (m0 + m) % RA
    long long a_m0, a_RA;
    long long B;                    // number of centres (rows of P and of centres)
    PassGeom pg;
    int out_mode;
    float* out;
    long long ld_out;
    float* cst;
    const float* centres;
    float eps;
    float* part;
    const float* col_bias;  // OUT_STORE only: added to every stored output column (nullptr: none)
    int count_const;
    int* err;
    int test_stall;  // test hook: CTA 0 never issues its first raw-tile copy, so a bounded wait expires
};

// Warp roles (11 warps): 0 raw-A/P producer + TMEM owner, 1 MMA issuer, 2-5 transform,
// 6-9 epilogue, 10 W producer.
constexpr int W_RAW = 0, W_MMA = 1, W_XF0 = 2, W_EPI0 = 6, W_B = 10;
static_assert(W_EPI0 - W_XF0 == 4 && W_B == W_EPI0 + 4, "four transform and four epilogue warps");

__global__ void __launch_bounds__(NUM_THREADS, 1)
dense_back_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
              const __grid_constant__ CUtensorMap tmBhi, const __grid_constant__ CUtensorMap tmBlo, TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bbytes = p.BN * BK * 4;
    const int pbytes = p.nbp * BK * 16;
    __shared__ uint64_t b_full[MAX_STAGES], b_empty[MAX_STAGES], r_full[MAX_STAGES], r_empty[MAX_STAGES];
    __shared__ uint64_t a_full[A_STAGES], a_empty[A_STAGES], acc_full, acc_empty, done_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BS = p.b_stages, RS = p.r_stages;
    const int nk = (p.K + BK - 1) / BK;
    const int ntn = p.ntiles_n;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < BS; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int s = 0; s < RS; ++s) {
            mbar_init(&r_full[s], 1);
            mbar_init(&r_empty[s], 128);
        }
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(&a_full[s], 128);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 128);
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == W_RAW) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int* abort_flag = &abort_sh;

    if (warp == W_RAW) {
        if (lane == 0) {
            // ------------------------------------------- raw coefficient tiles + relaxation slices
            long long g = 0;
            for (long long t = blockIdx.x; t < p.ntiles && !*abort_flag; t += gridDim.x) {
                const long long m_tile = t / ntn;
                const int ya = (p.a_row_mode == 0) ? (int)(m_tile * BM) : (int)((p.a_m0 + m_tile * BM) % p.a_RA);
                const int b_first = (int)((p.pg.pass_m0 + m_tile * BM) / p.pg.R_pass);
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int sr = (int)(g % RS);
                    if (g >= RS && !mbar_wait(&r_empty[sr], (uint32_t)((g / RS) - 1) & 1, abort_flag)) break;
                    if (p.test_stall && blockIdx.x == 0 && g == 0) continue;  // copy never issued (test hook)
                    mbar_expect_tx(&r_full[sr], TILE_A + pbytes);
                    tma_load_2d(base + p.r_off + sr * TILE_A, &tmA, &r_full[sr], kb * BK, ya);
                    tma_load_2d(base + p.p_off + sr * pbytes, &tmP, &r_full[sr], kb * BK * 4, b_first);
                }
            }
            if (*abort_flag)  // drain: wait (bounded) for copies nobody will consume
                for (long long h = (g > RS ? g - RS : 0); h < g; ++h) {
                    if (p.test_stall && blockIdx.x == 0 && h == 0) continue;  // never issued
                    const long long t0 = clock64();
                    while (!mbar_test(&r_full[h % RS], (uint32_t)(h / RS) & 1) && clock64() - t0 < WAIT_CYCLES) {
                    }
                }
        }
    } else if (warp == W_B) {
        if (lane == 0) {
            // ------------------------------------------------------------ W^T head/remainder tiles
            long long g = 0;
            for (long long t = blockIdx.x; t < p.ntiles && !*abort_flag; t += gridDim.x) {
                const int yb = (int)(t % ntn) * p.BN;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int sb = (int)(g % BS);
                    if (g >= BS && !mbar_wait(&b_empty[sb], (uint32_t)((g / BS) - 1) & 1, abort_flag)) break;
                    uint8_t* bst = base + p.b_off + (size_t)sb * 2 * bbytes;
                    mbar_expect_tx(&b_full[sb], 2 * bbytes);
                    tma_load_2d(bst, &tmBhi, &b_full[sb], kb * BK, yb);
                    tma_load_2d(bst + bbytes, &tmBlo, &b_full[sb], kb * BK, yb);
                }
            }
            if (*abort_flag)
                for (long long h = (g > BS ? g - BS : 0); h < g; ++h) {
                    const long long t0 = clock64();
                    while (!mbar_test(&b_full[h % BS], (uint32_t)(h / BS) & 1) && clock64() - t0 < WAIT_CYCLES) {
                    }
                }
        }
    } else if (warp == W_MMA) {
        if (lane == 0) {
            // ------------------------------------------------------------------------ MMA issuer
            const uint32_t idesc = idesc_tf32(BM, p.BN);
            long long g = 0, tiles_done = 0;
            for (long long t = blockIdx.x; t < p.ntiles && !*abort_flag; t += gridDim.x, ++tiles_done) {
                if (tiles_done > 0 && !mbar_wait(&acc_empty, (uint32_t)(tiles_done - 1) & 1, abort_flag)) break;
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int sa = (int)(g % A_STAGES), sb = (int)(g % BS);
                    if (!mbar_wait(&a_full[sa], (uint32_t)(g / A_STAGES) & 1, abort_flag)) break;
                    if (!mbar_wait(&b_full[sb], (uint32_t)(g / BS) & 1, abort_flag)) break;
                    tc_fence_after();
                    uint8_t* bst = base + p.b_off + (size_t)sb * 2 * bbytes;
                    const uint64_t db_hi = sw128_desc(smem_u32(bst));
                    const uint64_t db_lo = sw128_desc(smem_u32(bst + bbytes));
                    const uint32_t ta_hi = tmem + 256 + sa * 64;
                    const uint32_t ta_lo = ta_hi + 32;
#pragma unroll
                    for (int kk = 0; kk < BK / 8; ++kk) {
                        const uint64_t off = (uint64_t)(kk * 32) >> 4;  // 8 tf32 = 32 bytes along K in smem
                        const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                        mma_tf32_ts(tmem, ta_lo + kk * 8, db_hi + off, idesc, acc);
                        mma_tf32_ts(tmem, ta_hi + kk * 8, db_lo + off, idesc, 1u);
                        mma_tf32_ts(tmem, ta_hi + kk * 8, db_hi + off, idesc, 1u);
                    }
                    mma_commit(&a_empty[sa]);
                    mma_commit(&b_empty[sb]);
                }
                mma_commit(&acc_full);
            }
            // never free TMEM under MMAs still in flight, even after an abort: one last commit
            // tracks every MMA this thread issued
            mma_commit(&done_bar);
            const long long t0 = clock64();
            while (!mbar_test(&done_bar, 0) && clock64() - t0 < WAIT_CYCLES) {
            }
        }
    } else if (warp < W_EPI0) {
        // ------------------------------------------------------------------------- transform
        const int q = warp & 3;         // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;  // tile row owned by this thread (TMEM lane)
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        long long g = 0;
        for (long long t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
            const long long m_tile = t / ntn;
            const int n_tile = (int)(t % ntn);
            const long long m = m_tile * BM + row;
            const bool valid = m < p.M;
            const long long b = (p.pg.pass_m0 + m) / p.pg.R_pass;
            const long long b_first = (p.pg.pass_m0 + m_tile * BM) / p.pg.R_pass;
            const int cb = valid ? (int)(b - b_first) : 0;
            float cacc = 0.f;
            bool alive = true;
            for (int kb = 0; kb < nk; ++kb, ++g) {
                const int sr = (int)(g % RS), sa = (int)(g % A_STAGES);
                bool ok = mbar_wait(&r_full[sr], (uint32_t)(g / RS) & 1, abort_flag);
                float hi[32], lo[32];
                if (ok) {
                    const float4* arow = reinterpret_cast<const float4*>(base + p.r_off + sr * TILE_A + row * 128);
                    const float4* prow = reinterpret_cast<const float4*>(base + p.p_off + sr * pbytes) + cb * BK;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 x = arow[c ^ (row & 7)];  // 128-byte swizzle of the TMA tile
                        const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float4 pr = prow[c * 4 + j];
                            const float v = xv[j];
                            const float r = (v >= 0.f) ? v * pr.x : v * pr.y;
                            if (p.count_const) cacc = fmaf(fminf(v, 0.f), pr.z, cacc);
                            cacc = fmaf(r, pr.w, cacc);
                            const float h = tf32_hi(r);
                            hi[c * 4 + j] = h;
                            lo[c * 4 + j] = r - h;
                        }
                    }
                    mbar_arrive(&r_empty[sr]);
                    if (g >= A_STAGES) ok = mbar_wait(&a_empty[sa], (uint32_t)((g / A_STAGES) - 1) & 1, abort_flag);
                }
                if (!__all_sync(0xffffffffu, ok)) {
                    alive = false;
                    break;
                }
                const uint32_t ta = tmem + lane_base + 256 + sa * 64;
                tmem_st32(ta, hi);
                tmem_st32(ta + 32, lo);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                mbar_arrive(&a_full[sa]);
            }
            if (!alive) break;
            if (p.cst != nullptr && n_tile == 0 && valid) p.cst[m] += cacc;
        }
    } else {
        // -------------------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        float* stg = reinterpret_cast<float*>(base + p.s_off) + q * p.s_floats;
        long long tiles_done = 0;
        for (long long t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++tiles_done) {
            const long long m_tile = t / ntn;
            const int n_tile = (int)(t % ntn);
            const int n0 = n_tile * p.BN;
            const long long m = m_tile * BM + row;
            const bool valid = m < p.M;
            const long long row0 = m_tile * BM + q * 32;  // first row of this warp
            if (p.out_mode == OUT_CONCRETIZE) {
                // this warp's rows span centres bw .. bw + nbw - 1: stage their slice of the centres
                const long long bw = (p.pg.pass_m0 + row0) / p.pg.R_pass;
                for (int i = lane; i < p.nbw * p.BN; i += 32) {
                    const long long bb = bw + i / p.BN;
                    const int n = n0 + i % p.BN;
                    stg[i] = (bb < p.B && n < p.N) ? __ldg(&p.centres[bb * p.N + n]) : 0.f;
                }
                __syncwarp();
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full, (uint32_t)tiles_done & 1, abort_flag))) break;
            tc_fence_after();
            if (p.out_mode == OUT_CONCRETIZE) {
                const long long b = (p.pg.pass_m0 + m) / p.pg.R_pass;
                const long long bw = (p.pg.pass_m0 + row0) / p.pg.R_pass;
                const float* crow = stg + (valid ? (int)(b - bw) : 0) * p.BN;
                // sum_n v c_n and sum_n |v| over the tile's BN columns (BN is a multiple of 16): 64
                // columns in flight per wait, then a 32- and a 16-column tail
                float s1[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
                int c0 = 0;
                for (; c0 + 64 <= p.BN; c0 += 64) {
                    uint32_t v[2][32];
                    tmem_ld32_nowait(tmem + lane_base + c0, v[0]);
                    tmem_ld32_nowait(tmem + lane_base + c0 + 32, v[1]);
                    tmem_wait_ld();
                    conc_chunk<32>(v[0], crow + c0, s1, s2);
                    conc_chunk<32>(v[1], crow + c0 + 32, s1, s2);
                }
                if (c0 + 32 <= p.BN) {
                    uint32_t v[32];
                    tmem_ld32_nowait(tmem + lane_base + c0, v);
                    tmem_wait_ld();
                    conc_chunk<32>(v, crow + c0, s1, s2);
                    c0 += 32;
                }
                if (c0 < p.BN) {
                    uint32_t v[32];
                    tmem_ld16_nowait(tmem + lane_base + c0, v);
                    tmem_wait_ld();
                    conc_chunk<16>(v, crow + c0, s1, s2);
                }
                tc_fence_before();
                mbar_arrive(&acc_empty);
                const float conc = ((s1[0] + s1[1]) + (s1[2] + s1[3])) - p.eps * ((s2[0] + s2[1]) + (s2[2] + s2[3]));
                if (valid) p.part[(long long)n_tile * p.M + m] = conc;
                __syncwarp();  // the staged centres are reused by the next tile
            } else {
                // plain stores with 16-byte rows: each thread writes its own row's 32 columns as eight float4 (a short
                // drain, so the accumulator goes back to the MMA sooner); otherwise through a shared-memory transpose
                const bool vec = p.out_mode == OUT_STORE && (p.ld_out & 3) == 0 &&
                                 (reinterpret_cast<uintptr_t>(p.out) & 15) == 0 &&
                                 (p.col_bias == nullptr || (reinterpret_cast<uintptr_t>(p.col_bias) & 15) == 0);
                for (int c0 = 0; c0 < p.BN; c0 += 64) {
                    uint32_t v[2][32];
                    tmem_ld32_nowait(tmem + lane_base + c0, v[0]);
                    if (c0 + 32 < p.BN) tmem_ld32_nowait(tmem + lane_base + c0 + 32, v[1]);
                    tmem_wait_ld();
                    if (c0 + 64 >= p.BN) {  // accumulator fully read: hand TMEM back to the MMA
                        tc_fence_before();
                        mbar_arrive(&acc_empty);
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int cu = c0 + 32 * u;
                        if (cu >= p.BN) break;
                        if (vec && cu + 32 <= p.BN && n0 + cu + 32 <= p.N) {  // all 32 columns in the tile and the map
                            if (valid) {
                                float4* o4 = reinterpret_cast<float4*>(p.out + m * p.ld_out + n0 + cu);
                                const float4* b4 =
                                    p.col_bias != nullptr ? reinterpret_cast<const float4*>(p.col_bias + n0 + cu) : nullptr;
#pragma unroll
                                for (int q4 = 0; q4 < 8; ++q4) {
                                    const float4 bb = b4 != nullptr ? __ldg(&b4[q4]) : make_float4(0.f, 0.f, 0.f, 0.f);
                                    o4[q4] = make_float4(__uint_as_float(v[u][4 * q4]) + bb.x,
                                                         __uint_as_float(v[u][4 * q4 + 1]) + bb.y,
                                                         __uint_as_float(v[u][4 * q4 + 2]) + bb.z,
                                                         __uint_as_float(v[u][4 * q4 + 3]) + bb.w);
                                }
                            }
                            continue;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) stg[lane * 33 + j] = __uint_as_float(v[u][j]);
                        __syncwarp();
                        const int n = n0 + cu + lane;
                        const bool col_ok = (cu + lane < p.BN) && (n < p.N);
                        const float cb = (col_ok && p.col_bias != nullptr) ? __ldg(&p.col_bias[n]) : 0.f;
#pragma unroll 4
                        for (int j = 0; j < 32; ++j) {
                            const long long mr = row0 + j;
                            if (col_ok && mr < p.M) {
                                float* o = p.out + mr * p.ld_out + n;
                                const float val = stg[j * 33 + lane];
                                *o = (p.out_mode == OUT_ACCUM) ? (*o + val) : val + cb;
                            }
                        }
                        __syncwarp();
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_RAW) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
    if (threadIdx.x == 0 && abort_sh && p.err != nullptr) atomicExch(p.err, 1);
}

// ---------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {  // thread-safe one-time lookup
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// 2-D fp32 tensor map: inner dimension `cols` (contiguous), `rows` rows `ld` elements apart,
// box of box_cols x box_rows, 128-byte swizzle (box_cols = 32) or none, zero fill outside.
bool make_map(CUtensorMap* map, const float* ptr, long long cols, long long rows, long long ld, int box_rows,
              int box_cols, bool swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 4)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int pick_bn(int N, int* ntiles) {
    int t = (N + MAX_BN - 1) / MAX_BN;
    int bn = (N + t - 1) / t;
    bn = (bn + 15) / 16 * 16;
    *ntiles = (N + bn - 1) / bn;
    return bn;
}

// Centres a 128-row tile can span when a pass has R rows per centre.
long long centres_per_tile(long long R) { return 127 / R + 2; }

}  // namespace

int dense_back_tc_tiles_n(int N) {
    int t;
    pick_bn(N, &t);
    return t;
}

bool dense_back_tc_supported(const RowRef& A, Relax rx, long long M, int K, int N, PassGeom pg) {
    if (rx.P == nullptr) return false;                     // the bias rides in the relaxation table
    if (K % 4 != 0 || K < 32 || N < 16) return false;
    if (centres_per_tile(pg.R_pass) > 32) return false;
    if ((reinterpret_cast<uintptr_t>(A.ptr) & 15) != 0 || (A.ld % 4) != 0) return false;
    if (A.RA == kHugeRows && A.sB == 0 && A.m0 == 0) return M >= BM && M < (1LL << 31);  // chunk-local rows
    if (A.sB == 0 && A.RA % BM == 0 && A.m0 % BM == 0) return true;  // one block shared by all centres
    return false;
}

namespace {

cudaError_t launch_tc(const RowRef& A, Relax rx, const float* Wt_hi, const float* Wt_lo, long long B, long long M,
                     int K, int N, PassGeom pg, int out_mode, float* out, long long ld_out, float* cst,
                     const float* centres, float eps, float* part, const float* col_bias, int* err, int test_stall,
                     cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    TcParams p{};
    p.M = M;
    p.K = K;
    p.N = N;
    p.B = B;
    p.BN = pick_bn(N, &p.ntiles_n);
    p.nbp = (int)std::min<long long>(centres_per_tile(pg.R_pass), B);
    p.nbw = (int)std::min<long long>(31 / pg.R_pass + 2, B);
    p.ntiles = ((M + BM - 1) / BM) * p.ntiles_n;
    // epilogue staging per warp: a 32x33 block for stores, or the centre rows for concretisation
    p.s_floats = (out_mode == OUT_CONCRETIZE) ? p.nbw * p.BN : 32 * 33;
    const int sbytes = 4 * p.s_floats * 4;
    const int bstage = 2 * p.BN * BK * 4;
    const int rstage = TILE_A + p.nbp * BK * 16;
    const int budget = 220 * 1024 - 1024 - sbytes;
    p.b_stages = 2;
    p.r_stages = 2;
    while (p.b_stages < 4 && (p.b_stages + 1) * bstage + (p.r_stages + 1) * rstage <= budget) p.b_stages++;
    while (p.r_stages < MAX_STAGES && p.b_stages * bstage + (p.r_stages + 1) * rstage <= budget) p.r_stages++;
    if (p.b_stages * bstage + p.r_stages * rstage > budget) return cudaErrorInvalidValue;
    p.b_off = 0;
    p.r_off = p.b_stages * bstage;                        // multiple of 1024 (BN is a multiple of 16)
    p.p_off = p.r_off + p.r_stages * TILE_A;              // TILE_A is a multiple of 1024
    p.s_off = p.p_off + p.r_stages * p.nbp * BK * 16;     // multiple of 512
    const size_t smem = (size_t)p.s_off + sbytes + 1024;
    CUtensorMap ta, tp, tbh, tbl;
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
    if (!make_map(&ta, A.ptr, K, a_rows, A.ld, BM, 32, true) ||
        !make_map(&tp, reinterpret_cast<const float*>(rx.P), 4LL * K, B, 4LL * K, p.nbp, 128, false) ||
        !make_map(&tbh, Wt_hi, K, N, K, p.BN, 32, true) || !make_map(&tbl, Wt_lo, K, N, K, p.BN, 32, true))
        return cudaErrorInvalidValue;
    p.pg = pg;
    p.out_mode = out_mode;
    p.out = out;
    p.ld_out = ld_out;
    p.cst = cst;
    p.centres = centres;
    p.eps = eps;
    p.part = part;
    p.col_bias = col_bias;
    p.count_const = rx.count_const;
    p.err = err;
    p.test_stall = test_stall;
    cudaError_t e = allow_dyn_smem((const void*)dense_back_tc, 220 * 1024);
    if (e != cudaSuccess) return e;
    int dev = 0, num_sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long grid = std::min<long long>(p.ntiles, num_sms);  // persistent: one CTA per SM
    dense_back_tc<<<(unsigned)grid, NUM_THREADS, smem, s>>>(ta, tp, tbh, tbl, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dense_back_tc(const RowRef& A, Relax rx, const float* Wt_hi, const float* Wt_lo, long long B,
                                 long long M, int K, int N, PassGeom pg, int out_mode, float* out, long long ld_out,
                                 float* cst, const float* centres, float eps, float* part, int* err, int test_stall,
                                 cudaStream_t s) {
    return launch_tc(A, rx, Wt_hi, Wt_lo, B, M, K, N, pg, out_mode, out, ld_out, cst, centres, eps, part, nullptr,
                     err, test_stall, s);
}

bool dense_fwd_tc_supported(const float* A, long long M, int K, int N) {
    if (K % 4 != 0 || K < 32 || N < 16) return false;  // TMA rows of A and W: 16-byte strides
    if ((reinterpret_cast<uintptr_t>(A) & 15) != 0) return false;
    return M >= BM && M < (1LL << 31);
}

cudaError_t launch_dense_fwd_tc(const float* A, long long M, int K, int N, const float* W_hi, const float* W_lo,
                                const float* bias, const float4* ident, float* out, int* err, cudaStream_t s) {
    // the same kernel with every row read through one identity relaxation row (slopes 1, intercept 0, no row
    // constant) and the bias added per output column in the store epilogue
    return launch_tc(RowRef{A, 0, K, kHugeRows, 0}, Relax{ident, 0}, W_hi, W_lo, 1, M, K, N, PassGeom{0, kHugeRows},
                     OUT_STORE, out, N, nullptr, nullptr, 0.f, nullptr, bias, err, 0, s);
}

}  // namespace vf
