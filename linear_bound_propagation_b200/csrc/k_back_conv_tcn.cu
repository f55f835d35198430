// CROWN back-substitution through a convolution on the tensor cores with the taps in the N dimension
// (sm_100a, tcgen05.mma kind::tf32, 3xTF32): the same step as k_back_conv_tc.cu, organised so that each MMA is
// large. Selected with VF_CONV_TC=tapn. On the residual network it measures about 2x slower than the tap-shift
// kernel (the taps are summed one at a time through shared memory with a barrier per tap, and a group's staging,
// MMAs and tap sums run largely one after the other), so the tap-shift kernel is the default.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (the linear relaxation matrices A carried back through every layer),
// §2.1 (relaxation slopes from intermediate bounds) and §4.2-4.3 (CNN and ResNet models, BoundConv).
//
// For every row m, over the convolution output (co, oy, ox) in window wa:
//   r = relax(A[m, co, oy, ox]);  cst[m] += sum min(x, 0) t + r bias[co]
//   out[m, ci, s oy - pad + p, s ox - pad + q] += r W[co, ci, p, q]      for every tap (p, q)
// into the destination window wd (stored or accumulated), or concretised into cst.
//
// GEMM. M = coefficient positions (a, b) of the rows' windows (128 per MMA), K = output channels co (8 per MMA),
// N = (tap, ci) pairs: D[(a, b), (p, q, ci)] = sum_co r[co, a, b] W[co, ci, p, q]. The taps are summed afterwards:
// the output position of coefficient (a, b) under tap (p, q) is (s a + p, s b + q) in the natural window of the
// row (the receptive field of wa, origin (s aoy - pad, s aox - pad)); for one tap the map (a, b) -> output is one
// to one, so the epilogue adds one tap at a time into a shared-memory image of each row's natural window, taps in a
// fixed order, and writes the finished window out (stored, accumulated or concretised) with coalesced accesses.
// The taps are split into at most four groups of at most 256 columns (N_g = taps_g x C) that share one TMEM
// accumulator region per tile: columns [t ntot + col_g, + N_g).
//
// 3xTF32 (Ootomo & Yokota 2022 split): D = r_hi W_hi + r_hi W_lo + r_lo W_hi, three MMAs of N_g per group, tile
// and 8 channels into the same accumulator.
//
// Rows never straddle tiles: rows of npos = Ha Wa <= 128 positions are packed rpt = 128 / npos to a tile, larger
// rows take tpr = ceil(npos / 128) whole tiles. Each output therefore receives its contributions in an order fixed
// by the row's window size alone (tile by tile, tap by tap), whichever group and slot the row lands in.
//
// Roles (13 warps, one CTA per SM, persistent over groups of G rows):
//   warps 0-7:  stage each 8-channel chunk of the group's rows (gather, relax, split into head and remainder),
//               and sum the row constants per row in a fixed order;
//   warp 12:    one thread issues the MMAs (tap groups x parts x tiles per chunk) and commits;
//   warps 8-11: sum the taps into the rows' natural windows in shared memory (TMEM lane = coefficient position),
//               then write each row's window out and add its constant (and concretised sum) to cst.
// All mbarrier waits are bounded; a failed wait marks the warp dead, but every warp still walks its group loop,
// so the named barriers are always reached.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "conv_tc_common.cuh"
#include "tc_ptx.cuh"
#include "vf_internal.cuh"

namespace vf {

namespace {

using namespace tc;
using namespace conv_tc;

constexpr int BM = 128;
constexpr int XF_WARPS = 8;
constexpr int W_EPI0 = 8;
constexpr int W_MMA = 12;
constexpr int NUM_THREADS = 13 * 32;
constexpr int XF_THREADS = XF_WARPS * 32;
constexpr int MAX_G = 128;
constexpr int MAX_GROUPS = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_LIMIT = 220 * 1024;

struct ConvTcnParams {
    RowRef A;
    Relax rx;
    const float* bias;
    const float* Wtn;  // [chunk][group][part: head, remainder][2][N_g][4] floats
    long long M;
    ConvGeom g;
    PassGeom pg;
    PassStart ps;
    Win wa, wd;
    int C, nchunk, kk, ntot;              // input channels, 8-channel chunks, taps, TMEM columns per tile (C kk)
    int ngrp;
    int grp_tap0[MAX_GROUPS], grp_ntap[MAX_GROUPS], grp_col[MAX_GROUPS], grp_woff[MAX_GROUPS];
    int npos, rpt, tpr;                   // positions per row; rows per tile (packed) or tiles per row
    int G, T, NPOS;                       // rows per group, tiles per group, positions per stage (T * 128)
    int Hn, Wn, onat;                     // natural window and floats per row of it (C Hn Wn)
    int wpi, items;                       // staging warps per row, items per row and chunk
    int abuf, acc_cols;
    int w_resident, w_chunk_bytes;        // all chunks' weights resident, else one chunk per stage
    int a_stage_bytes, w_off, rc_off, rt_off, os_off, red_off;  // shared-memory plan
    float inv_plane, inv_wa, inv_npos, inv_hnwn, inv_wn;
    int out_mode;
    float* out;
    long long ld_out;
    float* cst;
    const float* centres;
    float eps;
    int* err;
};

// Flat stage position of (row slot i, window position pos).
__device__ __forceinline__ int row_base(const ConvTcnParams& p, int i) {
    return p.tpr > 1 ? i * p.tpr * BM : (i / p.rpt) * BM + (i % p.rpt) * p.npos;
}

// Stage U items for chunk c; item u belongs to row slot iu[u] with index eu[u] in the row: e = (4-channel half h,
// window position). The row's four coefficients of that half at that position are relaxed, split into tf32 head
// and remainder and written to the operand stage; the row-constant terms go to *csu[u].
template <int U>
__device__ __forceinline__ void stage_items(const ConvTcnParams& p, int c, const int (&iu)[U], const int (&eu)[U],
                                            const RowGeo* const (&rgu)[U], const float4* const (&Pbu)[U], int hw_o,
                                            uint8_t* sa, int stage_half, float* const (&csu)[U]) {
    const int Wa = p.wa.hw, plane_a = p.npos;
    float xv[U][4];
    float4 pr[U][4];
    int tpos[U], hh[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e = eu[u];
        live[u] = e < p.items;
        const int h = live[u] ? fdiv(e, p.inv_plane) : 0, pos = live[u] ? e - h * plane_a : 0;
        const int a = fdiv(pos, p.inv_wa), bb = pos - a * Wa;
        const int oy = rgu[u]->aoy + a, ox = rgu[u]->aox + bb;
        const bool on = live[u] && oy >= 0 && oy < p.g.ho && ox >= 0 && ox < p.g.wo;
        hh[u] = h;
        tpos[u] = row_base(p, iu[u]) + pos;
        const float* arow = rgu[u]->arow;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int co = 8 * c + 4 * h + j;
            const bool ld = on && co < p.g.co;
            xv[u][j] = ld ? __ldg(&arow[(long long)co * plane_a + pos]) : 0.f;
            pr[u][j] = (ld && Pbu[u] != nullptr) ? __ldg(&Pbu[u][(long long)co * hw_o + oy * p.g.wo + ox])
                                                 : make_float4(1.f, 1.f, 0.f, 0.f);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (!live[u]) continue;
        float r[4];
        float cs = *csu[u];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int co = 8 * c + 4 * hh[u] + j;
            const float x = xv[u][j];
            // off-map entries and padding channels hold x = 0, so they add nothing
            const float v = (x >= 0.f) ? x * pr[u][j].x : x * pr[u][j].y;
            if (p.rx.count_const) cs = fmaf(fminf(x, 0.f), pr[u][j].z, cs);
            if (p.bias != nullptr && co < p.g.co) cs = fmaf(v, __ldg(&p.bias[co]), cs);
            r[j] = v;
        }
        *csu[u] = cs;
        const float h0 = tf32_hi(r[0]), h1 = tf32_hi(r[1]), h2 = tf32_hi(r[2]), h3 = tf32_hi(r[3]);
        float4* hi = reinterpret_cast<float4*>(sa + (size_t)hh[u] * stage_half) + tpos[u];
        float4* lo = reinterpret_cast<float4*>(sa + (size_t)(2 + hh[u]) * stage_half) + tpos[u];
        *hi = make_float4(h0, h1, h2, h3);
        *lo = make_float4(r[0] - h0, r[1] - h1, r[2] - h2, r[3] - h3);
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) conv_back_tcn(const __grid_constant__ ConvTcnParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t a_full[2], a_empty[2], acc_full[2], acc_empty[2], rc_full[2], rc_empty[2], done_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ngroups = (p.M + p.G - 1) / p.G;
    float* rc = reinterpret_cast<float*>(base + p.rc_off);    // [2][G][wpi] row-constant partials
    RowGeo* rt = reinterpret_cast<RowGeo*>(base + p.rt_off);  // [2][G] row table, by group parity
    float* os = reinterpret_cast<float*>(base + p.os_off);    // [G][onat] the rows' natural windows
    float* red = reinterpret_cast<float*>(base + p.red_off);  // [G][4] concretised sums per row and epilogue warp

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(&a_full[s], XF_THREADS);
            mbar_init(&a_empty[s], 1);
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 128);
            mbar_init(&rc_full[s], XF_THREADS);
            mbar_init(&rc_empty[s], 128);
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (p.w_resident) {  // every chunk's weights, once
        const float4* src = reinterpret_cast<const float4*>(p.Wtn);
        float4* dst = reinterpret_cast<float4*>(base + p.w_off);
        const int nw4 = p.nchunk * p.w_chunk_bytes / 16;
        for (int i = threadIdx.x; i < nw4; i += NUM_THREADS) dst[i] = __ldg(&src[i]);
        fence_proxy_async_smem();
    }
    if (warp == W_EPI0) {
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
    const int stage_half = p.NPOS * 16;  // bytes of one 4-channel half of one (head or remainder) buffer

    if (warp < XF_WARPS) {
        // ------------------------------------------------------------------------------ staging
        const int ngrp_par = XF_WARPS / p.wpi;
        const int part = warp % p.wpi;
        const int tid = threadIdx.x;
        const long long nOut = (long long)p.g.co * p.g.ho * p.g.wo;
        const int hw_o = p.g.ho * p.g.wo;
        long long gc = 0;
        int it = 0;
        bool dead = false;
        for (long long q = blockIdx.x; q < ngroups; q += gridDim.x, ++it) {
            const long long m0 = q * p.G;
            const int rs = it & 1;
            if (!dead && it >= 2)
                dead = !__all_sync(0xffffffffu, mbar_wait(&rc_empty[rs], (uint32_t)((it >> 1) - 1) & 1, abort_flag));
            RowGeo* tab = rt + (size_t)rs * p.G;
            if (!dead)
                for (int i = tid; i < p.G; i += XF_THREADS)
                    if (m0 + i < p.M) tab[i] = row_geo(p, m0 + i);
            named_sync(2, XF_THREADS);  // the table is complete before any row is staged
            for (int c = 0; c < p.nchunk; ++c, ++gc) {
                const int st = (int)(gc & 1);
                if (!dead && gc >= 2)
                    dead = !__all_sync(0xffffffffu,
                                       mbar_wait(&a_empty[st], (uint32_t)((gc >> 1) - 1) & 1, abort_flag));
                if (dead) continue;
                uint8_t* sa = base + (size_t)st * 4 * stage_half;  // [head: 2 halves][remainder: 2 halves]
                if (!p.w_resident) {  // this chunk's weights
                    const float4* src = reinterpret_cast<const float4*>(p.Wtn) + (size_t)c * (p.w_chunk_bytes / 16);
                    float4* dst = reinterpret_cast<float4*>(base + p.w_off + (size_t)st * p.w_chunk_bytes);
                    for (int i = tid; i < p.w_chunk_bytes / 16; i += XF_THREADS) dst[i] = __ldg(&src[i]);
                }
                const int step = p.wpi * 32;
                const int e0 = part * 32 + lane;
                float* rcs = rc + (size_t)rs * p.G * p.wpi + part;
                if (p.items <= step) {
                    for (int i = warp / p.wpi; i < p.G; i += 2 * ngrp_par) {
                        if (m0 + i >= p.M) break;
                        const int i2 = i + ngrp_par;
                        const bool two = i2 < p.G && m0 + i2 < p.M;
                        float cs0 = 0.f, cs1 = 0.f;
                        const RowGeo* r0 = &tab[i];
                        const float4* P0 = p.rx.P != nullptr ? p.rx.P + r0->b * nOut : nullptr;
                        if (two) {
                            const RowGeo* r1 = &tab[i2];
                            const float4* P1 = p.rx.P != nullptr ? p.rx.P + r1->b * nOut : nullptr;
                            stage_items<2>(p, c, {i, i2}, {e0, e0}, {r0, r1}, {P0, P1}, hw_o, sa, stage_half,
                                           {&cs0, &cs1});
                        } else {
                            stage_items<1>(p, c, {i}, {e0}, {r0}, {P0}, hw_o, sa, stage_half, {&cs0});
                        }
                        cs0 = warp_sum32(cs0);
                        cs1 = warp_sum32(cs1);
                        if (lane == 0) {
                            rcs[(size_t)i * p.wpi] = (c == 0) ? cs0 : rcs[(size_t)i * p.wpi] + cs0;
                            if (two) rcs[(size_t)i2 * p.wpi] = (c == 0) ? cs1 : rcs[(size_t)i2 * p.wpi] + cs1;
                        }
                    }
                } else {
                    for (int i = warp / p.wpi; i < p.G; i += ngrp_par) {
                        if (m0 + i >= p.M) break;
                        const RowGeo* r0 = &tab[i];
                        const float4* P0 = p.rx.P != nullptr ? p.rx.P + r0->b * nOut : nullptr;
                        float cs = 0.f;
                        for (int e = e0; __any_sync(0xffffffffu, e < p.items); e += 2 * step) {
                            if (__any_sync(0xffffffffu, e + step < p.items))
                                stage_items<2>(p, c, {i, i}, {e, e + step}, {r0, r0}, {P0, P0}, hw_o, sa, stage_half,
                                               {&cs, &cs});
                            else
                                stage_items<1>(p, c, {i}, {e}, {r0}, {P0}, hw_o, sa, stage_half, {&cs});
                        }
                        cs = warp_sum32(cs);
                        if (lane == 0) rcs[(size_t)i * p.wpi] = (c == 0) ? cs : rcs[(size_t)i * p.wpi] + cs;
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&a_full[st]);
            }
            if (!dead) mbar_arrive(&rc_full[rs]);
        }
    } else if (warp == W_MMA) {
        // --------------------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t lbo_a = (uint32_t)stage_half;
            const uint64_t lo16 = (uint64_t)(2 * stage_half) >> 4;
            long long gc = 0;
            int it = 0;
            bool alive = true;
            for (long long q = blockIdx.x; q < ngroups && alive && !*abort_flag; q += gridDim.x, ++it) {
                const int ab = it % p.abuf;
                if (it >= p.abuf && !mbar_wait(&acc_empty[ab], (uint32_t)((it / p.abuf) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc0 = tmem + (uint32_t)(ab * p.acc_cols);
                for (int c = 0; c < p.nchunk; ++c, ++gc) {
                    const int st = (int)(gc & 1);
                    if (!mbar_wait(&a_full[st], (uint32_t)(gc >> 1) & 1, abort_flag)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = noswz_desc(smem_u32(base + (size_t)st * 4 * stage_half), lbo_a, 128);
                    const uint32_t wbase = smem_u32(base + p.w_off + (size_t)(p.w_resident ? c : st) * p.w_chunk_bytes);
                    for (int gi = 0; gi < p.ngrp; ++gi) {
                        const int ng = p.grp_ntap[gi] * p.C;
                        const uint32_t idesc = idesc_tf32(BM, ng);
                        const uint64_t b_hi = noswz_desc(wbase + (uint32_t)p.grp_woff[gi], (uint32_t)(ng * 16), 128);
                        const uint64_t b_lo = b_hi + (uint64_t)(ng * 2);  // + ng * 32 bytes
                        // head x W_hi, head x W_lo, remainder x W_hi; tiles innermost so consecutive MMAs go to
                        // different accumulators
#pragma unroll 1
                        for (int part = 0; part < 3; ++part) {
                            const uint64_t b = part == 1 ? b_lo : b_hi;
                            const uint64_t a0 = da + (part == 2 ? lo16 : 0);
                            const uint32_t acc = (c > 0 || part > 0) ? 1u : 0u;
                            for (int t = 0; t < p.T; ++t)
                                mma_tf32_ss(acc0 + (uint32_t)(t * p.ntot + p.grp_col[gi]), a0 + (uint64_t)(t * BM), b,
                                            idesc, acc);
                        }
                    }
                    mma_commit(&a_empty[st]);
                }
                if (!alive) break;
                mma_commit(&acc_full[ab]);
            }
            mma_commit(&done_bar);
            const long long t0 = clock64();
            while (!mbar_test(&done_bar, 0) && clock64() - t0 < WAIT_CYCLES) {
            }
        }
    } else {
        // ------------------------------------------------------------------------------ epilogue
        const int qd = warp & 3;
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        const int s = p.g.stride, k = p.g.k;
        const long long S_in = (long long)p.g.h * p.g.w;
        const int wdp = p.wd.hh * p.wd.hw;
        const int hnwn = p.Hn * p.Wn;
        const bool conc = p.out_mode == OUT_CONCRETIZE;
        const int etid = threadIdx.x - W_EPI0 * 32;  // 0..127
        int it = 0;
        bool dead = false;
        for (long long q = blockIdx.x; q < ngroups; q += gridDim.x, ++it) {
            const long long m0 = q * p.G;
            const int ab = it % p.abuf, rs = it & 1;
            const int grows = (int)std::min<long long>(p.G, p.M - m0);
            // clear the rows' natural windows (the previous group's write-out is complete)
            for (int e = etid; e < grows * p.onat; e += 128) os[e] = 0.f;
            if (!dead)
                dead = !__all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (uint32_t)(it / p.abuf) & 1, abort_flag));
            tc_fence_after();
            if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&rc_full[rs], (uint32_t)(it >> 1) & 1, abort_flag));
            named_sync(1, 128);  // windows cleared by every epilogue thread
            const RowGeo* tab = rt + (size_t)rs * p.G;
            const uint32_t acc0 = tmem + (uint32_t)(ab * p.acc_cols);
            // sum the taps into the natural windows: one tap at a time (a tap maps positions one to one)
            for (int t = 0; t < p.T; ++t) {
                const int u = qd * 32 + lane;  // coefficient position in tile t
                int i, pos;
                if (p.tpr > 1) {
                    i = t / p.tpr;
                    pos = (t - i * p.tpr) * BM + u;
                } else {
                    const int r = fdiv(u, p.inv_npos);
                    i = t * p.rpt + r;
                    pos = u - r * p.npos;
                    if (r >= p.rpt) pos = p.npos;  // past the tile's last row
                }
                const bool valid = !dead && i < grows && pos < p.npos;
                const int a = valid ? fdiv(pos, p.inv_wa) : 0, b = valid ? pos - a * p.wa.hw : 0;
                float* orow = os + (size_t)(valid ? i : 0) * p.onat;
                for (int gi = 0; gi < p.ngrp; ++gi)
                    for (int j = 0; j < p.grp_ntap[gi]; ++j) {
                        const int tap = p.grp_tap0[gi] + j;
                        const int pp = tap / k, qq = tap - pp * k;
                        const int y = s * a + pp, x = s * b + qq;
                        const uint32_t col = acc0 + (uint32_t)(t * p.ntot + p.grp_col[gi] + j * p.C);
                        for (int cb = 0; cb < p.C; cb += 16) {
                            uint32_t v[32];
                            __syncwarp();  // tcgen05.ld is warp-collective
                            if (!dead) {
                                tmem_ld16_nowait(lane_base + col + (uint32_t)cb, v);
                                tmem_wait_ld();
                            }
                            if (valid) {
                                float* o = orow + (size_t)cb * hnwn + y * p.Wn + x;
#pragma unroll
                                for (int jj = 0; jj < 16; ++jj) o[(size_t)jj * hnwn] += __uint_as_float(v[jj]);
                            }
                        }
                        named_sync(1, 128);  // the next tap may add to the same outputs
                    }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
            // write each row's natural window to its destination: all 128 epilogue threads on every row, four
            // elements per thread at a time with every load issued before the first store
            named_sync(1, 128);  // the tap sums of every thread are in the windows
            for (int i = 0; i < grows; ++i) {
                const long long m = m0 + i;
                const RowGeo rg = tab[i];
                const int noy = s * rg.aoy - p.g.pad, nox = s * rg.aox - p.g.pad;
                const float* orow = os + (size_t)i * p.onat;
                float* drow = conc ? nullptr : p.out + m * p.ld_out;
                const float* crow = conc ? p.centres + rg.b * (long long)p.C * S_in : nullptr;
                float sacc = 0.f;
                for (int e0 = etid; e0 < p.onat; e0 += 4 * 128) {
                    long long off[4];
                    bool on[4], in_wd[4];
                    float v[4], w[4];
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const int e = e0 + uu * 128;
                        const bool live = e < p.onat && !dead;
                        const int ci = live ? fdiv(e, p.inv_hnwn) : 0, rem = live ? e - ci * hnwn : 0;
                        const int cy = fdiv(rem, p.inv_wn), cx = rem - cy * p.Wn;
                        const int Y = noy + cy, X = nox + cx;
                        const int dy = Y - rg.doy, dx = X - rg.dox;
                        in_wd[uu] = live && dy >= 0 && dy < p.wd.hh && dx >= 0 && dx < p.wd.hw;
                        on[uu] = in_wd[uu] && Y >= 0 && Y < p.g.h && X >= 0 && X < p.g.w;
                        v[uu] = live ? orow[e] : 0.f;
                        if (conc) {
                            off[uu] = (long long)ci * S_in + (long long)Y * p.g.w + X;
                            w[uu] = on[uu] ? __ldg(&crow[off[uu]]) : 0.f;
                        } else {
                            off[uu] = (long long)ci * wdp + (long long)dy * p.wd.hw + dx;
                            w[uu] = (on[uu] && p.out_mode == OUT_ACCUM) ? drow[off[uu]] : 0.f;
                        }
                    }
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        if (conc) {
                            if (on[uu]) sacc += fmaf(v[uu], w[uu], -p.eps * fabsf(v[uu]));
                        } else if (in_wd[uu]) {
                            if (p.out_mode == OUT_ACCUM) {
                                if (on[uu]) drow[off[uu]] = w[uu] + v[uu];
                            } else {
                                drow[off[uu]] = on[uu] ? v[uu] : 0.f;
                            }
                        }
                    }
                }
                if (conc) {
                    sacc = warp_sum32(sacc);
                    if (lane == 0) red[(size_t)i * 4 + (warp - W_EPI0)] = sacc;
                }
            }
            named_sync(1, 128);  // every row's concretised partials are in red
            if (etid < grows && p.cst != nullptr && !dead) {
                float tot = 0.f;
                for (int w = 0; w < p.wpi; ++w) tot += rc[((size_t)rs * p.G + etid) * p.wpi + w];
                if (conc) tot += ((red[(size_t)etid * 4] + red[(size_t)etid * 4 + 1]) + red[(size_t)etid * 4 + 2]) +
                                 red[(size_t)etid * 4 + 3];
                p.cst[m0 + etid] += tot;
            }
            named_sync(1, 128);  // windows, constants and the table read before the next group uses them
            if (!dead) mbar_arrive(&rc_empty[rs]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_EPI0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
    if (threadIdx.x == 0 && abort_sh && p.err != nullptr) atomicExch(p.err, 1);
}

// Tap groups of at most 256 columns (N_g = taps x C, a multiple of 16); false when more than four are needed.
bool tap_groups(int C, int kk, ConvTcnParams* p) {
    const int per = std::max(1, 256 / C);  // taps per group
    p->ngrp = (kk + per - 1) / per;
    if (p->ngrp > MAX_GROUPS) return false;
    int col = 0, woff = 0;
    for (int g = 0; g < p->ngrp; ++g) {
        p->grp_tap0[g] = g * per;
        p->grp_ntap[g] = std::min(per, kk - g * per);
        p->grp_col[g] = col;
        p->grp_woff[g] = woff;
        col += p->grp_ntap[g] * C;
        woff += 2 * 2 * p->grp_ntap[g] * C * 16;  // head and remainder, two halves of 4 channels
    }
    p->ntot = col;
    return true;
}

bool plan_tcn(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode, ConvTcnParams* pp) {
    ConvTcnParams& p = *pp;
    if (g.ci % 16 != 0 || g.ci > 256 || g.k > 8) return false;
    p.C = g.ci;
    p.kk = g.k * g.k;
    p.nchunk = (g.co + 7) / 8;
    if (!tap_groups(p.C, p.kk, &p)) return false;
    if (p.ntot > (int)TMEM_COLS) return false;
    p.npos = wa.hh * wa.hw;
    p.Hn = g.stride * (wa.hh - 1) + g.k;
    p.Wn = g.stride * (wa.hw - 1) + g.k;
    p.onat = p.C * p.Hn * p.Wn;
    p.items = 2 * p.npos;
    const int vt = (p.items + 31) / 32;
    p.wpi = vt >= 8 ? 8 : (vt >= 4 ? 4 : (vt >= 2 ? 2 : 1));
    p.w_chunk_bytes = 2 * 2 * p.ntot * 16;  // all groups: head and remainder, two halves
    const int w_all = p.w_chunk_bytes * p.nchunk;
    p.w_resident = w_all <= 64 * 1024 ? 1 : 0;
    const int w_bytes = p.w_resident ? w_all : 2 * p.w_chunk_bytes;
    if (p.npos <= BM) {
        p.rpt = BM / p.npos;
        p.tpr = 1;
    } else {
        p.rpt = 1;
        p.tpr = (p.npos + BM - 1) / BM;
    }
    // two accumulator sets only when each still holds four tiles: with fewer, the per-group waits and barriers
    // cost more than the overlap of the (short) MMAs with the epilogue gains
    for (int abuf = 2; abuf >= 1; --abuf) {
        const int cols = (int)TMEM_COLS / abuf;
        const int tmax = cols / p.ntot;
        if (tmax < p.tpr || (abuf == 2 && tmax < 4)) continue;
        for (int T = (p.tpr > 1 ? p.tpr : tmax); T >= 1; --T) {
            const int G = p.tpr > 1 ? 1 : std::min(MAX_G, T * p.rpt);
            const int NPOS = T * BM;
            const int a_stage = 4 * NPOS * 16;
            const int rc_bytes = 2 * G * p.wpi * 4;
            const int rt_bytes = 2 * G * (int)sizeof(RowGeo);
            const int os_bytes = G * p.onat * 4;
            const int total = 2 * a_stage + w_bytes + ((rc_bytes + 15) / 16 * 16) + ((rt_bytes + 63) / 64 * 64) +
                              os_bytes + G * 16 + 1024;
            if (total > SMEM_LIMIT) continue;
            p.G = G;
            p.T = p.tpr > 1 ? p.tpr : (G + p.rpt - 1) / p.rpt;
            p.NPOS = p.T * BM;
            p.abuf = abuf;
            p.acc_cols = cols;
            p.a_stage_bytes = 2 * (4 * p.NPOS * 16);
            p.w_off = p.a_stage_bytes;
            p.rc_off = p.w_off + w_bytes;
            p.rt_off = p.rc_off + (rc_bytes + 15) / 16 * 16;
            p.os_off = p.rt_off + (rt_bytes + 63) / 64 * 64;
            p.red_off = p.os_off + os_bytes;
            p.inv_plane = 1.f / (float)p.npos;
            p.inv_wa = 1.f / (float)wa.hw;
            p.inv_npos = 1.f / (float)p.npos;
            p.inv_hnwn = 1.f / (float)(p.Hn * p.Wn);
            p.inv_wn = 1.f / (float)p.Wn;
            return true;
        }
    }
    return false;
}

size_t smem_bytes_tcn(const ConvTcnParams& p) { return (size_t)p.red_off + (size_t)p.G * 16 + 1024; }

}  // namespace

int conv_tcn_wtn_floats(const ConvGeom& g) {
    ConvTcnParams p{};
    if (g.ci % 16 != 0 || !tap_groups(g.ci, g.k * g.k, &p)) return 0;
    return ((g.co + 7) / 8) * 2 * 2 * p.ntot * 4;
}

void conv_tcn_pack_weights(const ConvGeom& g, const float* W, float* out) {
    ConvTcnParams p{};
    tap_groups(g.ci, g.k * g.k, &p);
    const int C = g.ci, nchunk = (g.co + 7) / 8;
    size_t o = 0;
    for (int c = 0; c < nchunk; ++c)
        for (int gi = 0; gi < p.ngrp; ++gi) {
            const int ng = p.grp_ntap[gi] * C;
            for (int part = 0; part < 2; ++part)
                for (int hk = 0; hk < 2; ++hk)
                    for (int n = 0; n < ng; ++n)
                        for (int j = 0; j < 4; ++j) {
                            const int tap = p.grp_tap0[gi] + n / C, ci = n % C;
                            const int pp = tap / g.k, qq = tap % g.k;
                            const int co = 8 * c + 4 * hk + j;
                            float w = 0.f;
                            if (co < g.co) w = W[(((size_t)co * g.ci + ci) * g.k + pp) * g.k + qq];
                            uint32_t bits;
                            std::memcpy(&bits, &w, 4);
                            bits &= 0xFFFFE000u;
                            float hi;
                            std::memcpy(&hi, &bits, 4);
                            out[o++] = part == 0 ? hi : w - hi;
                        }
        }
}

bool conv_back_tcn_supported(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode) {
    ConvTcnParams p{};
    return plan_tcn(g, wa, wd, out_mode, &p);
}

cudaError_t launch_conv_back_tcn(const RowRef& A, Relax rx, const float* Wtn, const float* bias, long long M,
                                 const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                 int out_mode, float* out, long long ld_out, float* cst, const float* centres,
                                 float eps, int* err, int num_sms, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    ConvTcnParams p{};
    if (!plan_tcn(g, wa, wd, out_mode, &p)) return cudaErrorInvalidValue;
    p.A = A;
    p.rx = rx;
    p.bias = bias;
    p.Wtn = Wtn;
    p.M = M;
    p.g = g;
    p.pg = pg;
    p.ps = ps;
    p.wa = wa;
    p.wd = wd;
    p.out_mode = out_mode;
    p.out = out;
    p.ld_out = ld_out;
    p.cst = cst;
    p.centres = centres;
    p.eps = eps;
    p.err = err;
    const size_t smem = smem_bytes_tcn(p);
    cudaError_t e = allow_dyn_smem((const void*)conv_back_tcn, SMEM_LIMIT + 1024);
    if (e != cudaSuccess) return e;
    const long long ngroups = (M + p.G - 1) / p.G;
    const long long grid = std::min<long long>(ngroups, num_sms);
    static const bool trace = getenv("VF_TRACE_CONV_TC") != nullptr;
    if (trace)  // launch plan, for profiling
        fprintf(stderr,
                "conv_back_tcn M=%lld ci=%d co=%d k=%d s=%d wa=%dx%d wd=%dx%d mode=%d G=%d T=%d ngrp=%d ntot=%d abuf=%d "
                "smem=%zu groups=%lld\n",
                M, g.ci, g.co, g.k, g.stride, wa.hh, wa.hw, wd.hh, wd.hw, out_mode, p.G, p.T, p.ngrp, p.ntot, p.abuf,
                smem, ngroups);
    conv_back_tcn<<<(unsigned)grid, NUM_THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace vf
