// CROWN back-substitution through a convolution on the 5th-generation tensor cores (sm_100a): the
// transposed convolution of relaxed coefficient rows as an implicit GEMM, tcgen05.mma kind::tf32 with the
// 3xTF32 split, operands in shared memory, accumulators in TMEM.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (the linear relaxation matrices A carried back through every layer),
// §2.1 (relaxation slopes from intermediate bounds) and §4.2-4.3 (CNN and ResNet models, BoundConv).
//
// For every row m, over the convolution output (co, oy, ox) in window wa (the whole map, or a receptive-field
// window whose origin depends on the row's start neuron):
//   r      = relax(A[m, co, oy, ox])                   (x * lo if x >= 0 else x * up, per centre and neuron)
//   cst[m] += sum min(x, 0) * t + r * bias[co]
//   out[m, ci, y, x] (=, +=) sum over (co, p, q) with y = s*oy - pad + p, x = s*ox - pad + q of r * W[co, ci, p, q]
// or, concretised, cst[m] += sum over on-map (ci, y, x) of out * c_b - eps * |out|.
//
// Implicit GEMM by tap shifts. The input positions split into s*s stride classes (y mod s, x mod s); within a
// class every output position gets the same taps, each reading the coefficient map at a fixed offset. The
// relaxed rows of G rows ("images") are laid out in shared memory as one flat sequence of slabs of S = Ha + g
// lines of pitch P = Wa + g (g = ceil(k/s) - 1 zero lines and columns in front of the data), so a tap is a
// constant shift of the flat position index: for output positions u of a class the GEMM operand of tap
// (p, q) = (s jy + ry, s jx + rx) is the flat rows u + (g - jy) P + (g - jx), which stay inside the row's own
// slab or the zero gap after it. The K dimension is the output channels, 8 per MMA; the N dimension the
// input channels. Per output position the slab coordinates (c', d') of class (ry, rx) give the natural
// window coordinates (s c' + ry, s d' + rx) relative to (s aoy - pad, s aox - pad).
//
// 3xTF32 in two MMAs (Ootomo & Yokota 2022 split, regrouped): with r = r_hi + r_lo and W = W_hi + W_lo,
//   D[:, 0:C)  = r_hi W_hi + r_lo W_hi        D[:, C:2C) = r_hi W_lo
// one MMA of N = 2C on r_hi against [W_hi | W_lo] and one of N = C on r_lo against W_hi; the epilogue adds
// the two halves. Each shared-memory operand row is read twice per tap instead of three times.
//
// Shared-memory layout (no swizzle, K-major): an operand row (one flat position, 4 channels) is 16 bytes;
// 8-row groups are contiguous (SBO = 128 B) and the two 4-channel halves of an 8-channel K step are NPOS rows
// apart (LBO = 16 NPOS B), so moving an operand by d rows moves its start address by 16 d bytes.
//
// Roles in a CTA of 13 warps (one CTA per SM, persistent over groups of G rows):
//   warps 0-7:  stage the 8-channel chunks of the group's rows: gather, relax, split into tf32 head and
//               remainder, write both into a shared-memory stage (two stages), copy the chunk's weights;
//               sum the row constants (per row, in an order that depends only on the window size);
//   warps 8-11: epilogue: read the accumulators (TMEM lane = flat position), add the two halves, store,
//               accumulate or concretise each row's outputs, and add the row's constant to cst;
//   warp 12:    one thread issues the MMAs and commits each chunk and each group.
// TMEM: 512 columns, one or two accumulator sets. All waits are bounded: on expiry a shared abort flag stops
// every role, the MMA thread waits (bounded) for its MMAs, TMEM is freed and the kernel reports through *err.
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
constexpr int MAX_TAPS = 64;
constexpr int MAX_G = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_LIMIT = 220 * 1024;

struct ConvTcParams {
    RowRef A;
    Relax rx;
    const float* bias;
    const float* Wtc;  // [k*k][nchunk][2][Np][4] floats: per tap and 8-channel chunk, the B operand image
    long long M;
    ConvGeom g;
    PassGeom pg;
    PassStart ps;
    Win wa, wd;
    int C, Np, nchunk;        // input channels padded to a multiple of 16 (N), 2C, output-channel chunks of 8 (K)
    int Cr;                   // input channels of the map (C_in; the channels from Cr to C carry zero weights)
    int G, S, P, gy, gx;      // rows per group, slab lines, pitch, gap lines / columns
    int npos_img, T, NPOS;    // flat positions per row, M tiles per class, positions per stage buffer
    int ncls, nact;           // s*s classes, classes with at least one tap
    int cls_ry[4], cls_rx[4], cls_nt[4], cls_t0[4];  // classes, active ones first
    int tap_shift[MAX_TAPS], tap_w[MAX_TAPS];
    int Hn, Wn;               // natural window (receptive field of wa) size
    int wpi, items;           // warps per row in the staging, staging items per row and chunk
    int abuf, acc_cols;       // accumulator sets, TMEM columns per set
    int a_stage_bytes, w_stage_bytes, w_off, rc_off, rt_off, cp_off;  // shared-memory plan
    int w_resident;  // 1: every chunk's weights loaded once per CTA (w region = all of Wtc), else per chunk
    float inv_plane, inv_wa, inv_npos, inv_p;  // 1 / (Ha Wa), 1 / Wa, 1 / npos_img, 1 / P (exact quotients, fdiv)
    int out_mode;
    float* out;
    long long ld_out;
    float* cst;
    const float* centres;
    float eps;
    int* err;
};

// One block of 16 input channels (cb .. cb + 15) of one flat position: the accumulator columns of the head
// half [cb, cb + 16) and of the remainder half [C + cb, C + cb + 16), added and then stored, accumulated or
// concretised. Warp-collective (tcgen05.ld).
__device__ __forceinline__ void epi_block16(const ConvTcParams& p, bool act, bool wr, bool on, bool conc,
                                            uint32_t col0, int cb, float* orow, const float* crow, int wdp,
                                            long long S_in, float* cpart) {
    uint32_t vh[32], vl[32];
    __syncwarp();
    if (act) {
        tmem_ld16_nowait(col0 + (uint32_t)cb, vh);
        tmem_ld16_nowait(col0 + (uint32_t)(p.C + cb), vl);
        tmem_wait_ld();
    }
    if (!wr) return;
    const int nc = min(16, p.Cr - cb);  // channels of the map in this block (padding channels are not written)
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = act ? __uint_as_float(vh[j]) + __uint_as_float(vl[j]) : 0.f;
    if (conc) {  // all the block's centre loads in flight at once
        float cv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) cv[j] = (on && j < nc) ? __ldg(&crow[(long long)(cb + j) * S_in]) : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < nc) acc += fmaf(v[j], cv[j], -p.eps * fabsf(v[j]));
        *cpart += acc;
    } else if (p.out_mode == OUT_ACCUM) {  // read all the block's old values before the first store
        if (!on) return;
        float old[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) old[j] = j < nc ? orow[(long long)(cb + j) * wdp] : 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < nc) orow[(long long)(cb + j) * wdp] = old[j] + v[j];
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < nc) orow[(long long)(cb + j) * wdp] = on ? v[j] : 0.f;
    }
}

// Stage U items for output-channel chunk c; item u belongs to row slot iu[u] (table entry rgu[u], relaxation
// base Pbu[u]) and has index eu[u] in that row: e = (4-channel half h, window position). Each holds the row's
// four coefficients of that half at that position, relaxed, split into tf32 head and remainder and written to
// the operand stage `sa`; its row-constant terms go to *csu[u]. Items at or past p.items are skipped. All loads
// of the U items are issued before any is used.
template <int U>
__device__ __forceinline__ void stage_items(const ConvTcParams& p, int c, const int (&iu)[U], const int (&eu)[U],
                                            const RowGeo* const (&rgu)[U], const float4* const (&Pbu)[U], int hw_o,
                                            uint8_t* sa, int stage_half, float* const (&csu)[U]) {
    const int Wa = p.wa.hw, plane_a = p.wa.hh * p.wa.hw;
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
        tpos[u] = iu[u] * p.npos_img + (p.gy + a) * p.P + (p.gx + bb);
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

__global__ void __launch_bounds__(NUM_THREADS, 1) conv_back_tc(const __grid_constant__ ConvTcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t a_full[2], a_empty[2], acc_full[2], acc_empty[2], rc_full[2], rc_empty[2], done_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ uint32_t tap_a16[MAX_TAPS], tap_b16[MAX_TAPS];  // per tap: operand offsets in 16-byte units

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ngroups = (p.M + p.G - 1) / p.G;
    float* rc = reinterpret_cast<float*>(base + p.rc_off);  // [2][G][wpi] row-constant partials
    float* cp = reinterpret_cast<float*>(base + p.cp_off);  // [nact * T * 128] concretised per position
    RowGeo* rt = reinterpret_cast<RowGeo*>(base + p.rt_off);  // [2][G] row table, by group parity

    if (threadIdx.x < MAX_TAPS) {
        const int tap = threadIdx.x;
        tap_a16[tap] = (uint32_t)p.tap_shift[tap];
        // B operand of tap w (chunk 0): resident weights are [tap][chunk][2 Np 4], a chunk stage [tap][2 Np 4]
        tap_b16[tap] = (uint32_t)(p.tap_w[tap] * (p.w_resident ? p.nchunk : 1) * p.Np * 2);
    }
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
    // zero both operand stages once: the gap lines and columns of every slab are never written again
    {
        float4* z = reinterpret_cast<float4*>(base);
        const int n4 = p.a_stage_bytes / 16;  // two stages, each hi and lo, back to back
        for (int i = threadIdx.x; i < n4; i += NUM_THREADS) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.w_resident) {  // every chunk's weights, once
            const float4* src = reinterpret_cast<const float4*>(p.Wtc);
            float4* dst = reinterpret_cast<float4*>(base + p.w_off);
            const int nw4 = p.g.k * p.g.k * p.nchunk * p.Np * 2;
            for (int i = threadIdx.x; i < nw4; i += NUM_THREADS) dst[i] = __ldg(&src[i]);
        }
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
    const int stage_half = p.NPOS * 16;  // bytes of one 4-channel half of one (hi or lo) buffer

    if (warp < XF_WARPS) {
        // ------------------------------------------------------------------------------ staging
        const int ngrp_par = XF_WARPS / p.wpi;  // rows staged at once
        const int part = warp % p.wpi;
        const int tid = threadIdx.x;
        const long long nOut = (long long)p.g.co * p.g.ho * p.g.wo;
        const int hw_o = p.g.ho * p.g.wo;
        long long gc = 0;
        int it = 0;
        // A failed (bounded) wait makes the warp dead: it skips all further work but keeps walking the
        // group loop, so the named barrier below is always reached by all staging warps.
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
                uint8_t* sa = base + (size_t)st * 2 * 2 * stage_half;  // [hi: 2 halves][lo: 2 halves]
                // this chunk's weights, every tap (unless all chunks are resident)
                if (!p.w_resident) {
                    const int per_tap4 = p.Np * 2;  // float4 per tap: [2][Np][4]
                    const float4* src = reinterpret_cast<const float4*>(p.Wtc);
                    float4* dst = reinterpret_cast<float4*>(base + p.w_off + (size_t)st * p.w_stage_bytes);
                    const int kk = p.g.k * p.g.k;
                    for (int i = tid; i < kk * per_tap4; i += XF_THREADS) {
                        const int tap = i / per_tap4, e = i - tap * per_tap4;
                        dst[i] = __ldg(&src[((size_t)tap * p.nchunk + c) * per_tap4 + e]);
                    }
                }
                const int step = p.wpi * 32;
                const int e0 = part * 32 + lane;
                float* rcs = rc + (size_t)rs * p.G * p.wpi + part;
                if (p.items <= step) {
                    // one item per lane and row: two rows at a time, so sixteen loads are in flight per lane
                    for (int i = warp / p.wpi; i < p.G; i += 2 * ngrp_par) {
                        if (m0 + i >= p.M) break;
                        const int i2 = i + ngrp_par;
                        const bool two = i2 < p.G && m0 + i2 < p.M;
                        float cs0 = 0.f, cs1 = 0.f;
                        if (two) {
                            const RowGeo* r0 = &tab[i];
                            const RowGeo* r1 = &tab[i2];
                            const float4* P0 = p.rx.P != nullptr ? p.rx.P + r0->b * nOut : nullptr;
                            const float4* P1 = p.rx.P != nullptr ? p.rx.P + r1->b * nOut : nullptr;
                            stage_items<2>(p, c, {i, i2}, {e0, e0}, {r0, r1}, {P0, P1}, hw_o, sa, stage_half,
                                           {&cs0, &cs1});
                        } else {
                            const RowGeo* r0 = &tab[i];
                            const float4* P0 = p.rx.P != nullptr ? p.rx.P + r0->b * nOut : nullptr;
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
                        // two items of the row per lane and iteration while it has them, then one
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
            const uint32_t id_full = idesc_tf32(BM, p.Np), id_half = idesc_tf32(BM, p.C);
            const uint32_t lbo_a = (uint32_t)stage_half, lbo_b = (uint32_t)(p.Np * 16);
            const uint64_t lo16 = (uint64_t)(2 * stage_half) >> 4;  // head -> remainder buffer, 16-byte units
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
                    // descriptors of this stage; a tap or tile moves only the 14-bit start-address field (the
                    // shared-memory window is below 256 KB, so the sum never carries out of it)
                    const uint64_t da = noswz_desc(smem_u32(base + (size_t)st * 2 * 2 * stage_half), lbo_a, 128);
                    const uint64_t db =
                        p.w_resident ? noswz_desc(smem_u32(base + p.w_off), lbo_b, 128) + (uint64_t)(c * p.Np * 2)
                                     : noswz_desc(smem_u32(base + p.w_off + (size_t)st * p.w_stage_bytes), lbo_b, 128);
                    // taps outermost, tiles innermost: consecutive MMAs go to different accumulators, so
                    // they overlap in the tensor pipe instead of each waiting for the previous one's result
                    for (int k = 0; k < p.nact; ++k) {
                        const int t0 = p.cls_t0[k], nt = p.cls_nt[k];
                        const uint32_t dk = acc0 + (uint32_t)(k * p.T * p.Np);
                        for (int j = 0; j < nt; ++j) {
                            const uint64_t a_tap = da + tap_a16[t0 + j];
                            const uint64_t b = db + tap_b16[t0 + j];
                            const uint32_t acc = (c > 0 || j > 0) ? 1u : 0u;
                            for (int t = 0; t < p.T; ++t)
                                mma_tf32_ss(dk + (uint32_t)(t * p.Np), a_tap + (uint64_t)(t * BM), b, id_full, acc);
                            for (int t = 0; t < p.T; ++t)
                                mma_tf32_ss(dk + (uint32_t)(t * p.Np), a_tap + (uint64_t)(t * BM) + lo16, b, id_half, 1u);
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
        const int qd = warp & 3;  // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
        const int s = p.g.stride;
        const long long S_in = (long long)p.g.h * p.g.w;
        const int wdp = p.wd.hh * p.wd.hw;
        const bool conc = p.out_mode == OUT_CONCRETIZE;
        int it = 0;
        bool dead = false;  // as in the staging warps: skip work after a failed wait, still reach the barriers
        for (long long q = blockIdx.x; q < ngroups; q += gridDim.x, ++it) {
            const long long m0 = q * p.G;
            const int ab = it % p.abuf, rs = it & 1;
            if (!dead)
                dead = !__all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (uint32_t)(it / p.abuf) & 1, abort_flag));
            tc_fence_after();
            // the staging of this group is complete: its row table and row constants are in shared memory
            if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&rc_full[rs], (uint32_t)(it >> 1) & 1, abort_flag));
            if (dead) {
                named_sync(1, 128);
                named_sync(1, 128);
                continue;
            }
            const RowGeo* tab = rt + (size_t)rs * p.G;
            const uint32_t acc0 = tmem + (uint32_t)(ab * p.acc_cols);
            for (int k = 0; k < p.ncls; ++k) {
                const bool act = k < p.nact;
                const int ry = p.cls_ry[k], rx = p.cls_rx[k];
                for (int t = 0; t < p.T; ++t) {
                    const int u = t * BM + qd * 32 + lane;  // this thread's flat position of class k
                    const int i = fdiv(u, p.inv_npos);
                    const int tt = u - i * p.npos_img;
                    const int c1 = fdiv(tt, p.inv_p), d1 = tt - c1 * p.P;
                    const int cy = s * c1 + ry, cx = s * d1 + rx;  // natural window coordinates
                    const long long m = m0 + i;
                    const bool valid = i < p.G && m < p.M && cy < p.Hn && cx < p.Wn;
                    RowGeo rg{0, 0, 0, 0, 0, nullptr};
                    int Y = -1, X = -1, dy = 0, dx = 0;
                    bool on = false, in_wd = false;
                    if (valid) {
                        rg = tab[i];
                        Y = s * rg.aoy - p.g.pad + cy;
                        X = s * rg.aox - p.g.pad + cx;
                        dy = Y - rg.doy;
                        dx = X - rg.dox;
                        in_wd = dy >= 0 && dy < p.wd.hh && dx >= 0 && dx < p.wd.hw;
                        on = in_wd && Y >= 0 && Y < p.g.h && X >= 0 && X < p.g.w;
                    }
                    // on-map outputs are written (or concretised); a STORE also writes zeros at the window's
                    // off-map entries
                    const bool wr = on || (in_wd && p.out_mode == OUT_STORE);
                    float* orow = (valid && !conc) ? p.out + m * p.ld_out + (long long)dy * p.wd.hw + dx : nullptr;
                    const float* crow = (valid && conc) ? p.centres + rg.b * (long long)p.Cr * S_in + (long long)Y * p.g.w + X
                                                        : nullptr;
                    float cpart = 0.f;
                    const uint32_t col0 = lane_base + acc0 + (uint32_t)((k * p.T + t) * p.Np);
                    float* ob = orow;
                    const float* cb_ = crow;
                    for (int cb = 0; cb < p.C; cb += 16)
                        epi_block16(p, act, wr, on, conc, col0, cb, ob, cb_, wdp, S_in, &cpart);
                    if (conc && act) cp[(size_t)(k * p.T + t) * BM + qd * 32 + lane] = cpart;
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
            named_sync(1, 128);  // every epilogue thread's concretised partials are in shared memory
            // per row: its concretised positions (classes in order, slab positions in order) and its constant
            for (int i = warp - W_EPI0; i < p.G; i += 4) {
                const long long m = m0 + i;
                if (m >= p.M) break;
                float sacc = 0.f;
                if (conc)
                    for (int k = 0; k < p.nact; ++k)
                        for (int tt = lane; tt < p.npos_img; tt += 32)
                            sacc += cp[(size_t)k * p.T * BM + (size_t)i * p.npos_img + tt];
                sacc = warp_sum32(sacc);
                if (lane == 0 && p.cst != nullptr) {
                    float tot = 0.f;
                    for (int w = 0; w < p.wpi; ++w) tot += rc[((size_t)rs * p.G + i) * p.wpi + w];
                    p.cst[m] += tot + sacc;
                }
            }
            named_sync(1, 128);  // partials and constants read before the next group writes them
            mbar_arrive(&rc_empty[rs]);
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

}  // namespace

// ---------------------------------------------------------------------------------------- host side

int conv_tc_wtc_floats(const ConvGeom& g) {
    const int nchunk = (g.co + 7) / 8, C = (g.ci + 15) / 16 * 16;
    return g.k * g.k * nchunk * 2 * (2 * C) * 4;
}

void conv_tc_pack_weights(const ConvGeom& g, const float* W, float* out) {
    const int C = (g.ci + 15) / 16 * 16, Np = 2 * C, nchunk = (g.co + 7) / 8;
    for (int p = 0; p < g.k; ++p)
        for (int q = 0; q < g.k; ++q)
            for (int c = 0; c < nchunk; ++c)
                for (int hk = 0; hk < 2; ++hk)
                    for (int n = 0; n < Np; ++n)
                        for (int j = 0; j < 4; ++j) {
                            const int co = 8 * c + 4 * hk + j, ci = n % C;
                            float w = 0.f;
                            if (co < g.co && ci < g.ci) w = W[(((size_t)co * g.ci + ci) * g.k + p) * g.k + q];
                            uint32_t bits;
                            std::memcpy(&bits, &w, 4);
                            bits &= 0xFFFFE000u;
                            float hi;
                            std::memcpy(&hi, &bits, 4);
                            out[((((size_t)(p * g.k + q) * nchunk + c) * 2 + hk) * Np + n) * 4 + j] = (n < C) ? hi : w - hi;
                        }
}

bool conv_tc_weights_supported(const ConvGeom& g) {
    // input channels a multiple of 16, or fewer than 16 at stride 1 (padded to 16 with zero weights: an MMA costs
    // the same at N = 2 x 16 as at N = 2 x 3, so a 3-channel 3x3 stem runs like a 16-channel convolution, faster than
    // the FFMA kernels on the residual network; the 4x4 stride-2 stem of the CNN measured slower than its windowed
    // FFMA kernel and stays there)
    return (g.ci % 16 == 0 || (g.ci < 16 && g.stride == 1)) && g.ci <= 128 && g.k <= 8 && g.stride >= 1 &&
           g.stride <= 2 && g.k * g.k <= MAX_TAPS;
}

namespace {

bool plan(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode, ConvTcParams* pp) {
    if (!conv_tc_weights_supported(g)) return false;
    ConvTcParams& p = *pp;
    const int s = g.stride, KS = (g.k + s - 1) / s;
    p.C = (g.ci + 15) / 16 * 16;
    p.Cr = g.ci;
    p.Np = 2 * p.C;
    p.nchunk = (g.co + 7) / 8;
    p.gy = p.gx = KS - 1;
    p.S = wa.hh + p.gy;
    p.P = wa.hw + p.gx;
    p.npos_img = p.S * p.P;
    p.Hn = s * (wa.hh - 1) + g.k;
    p.Wn = s * (wa.hw - 1) + g.k;
    p.ncls = s * s;
    // classes with taps first, then the empty ones (their outputs are zero)
    int ntap = 0, k = 0;
    for (int pass = 0; pass < 2; ++pass)
        for (int ry = 0; ry < s; ++ry)
            for (int rx = 0; rx < s; ++rx) {
                const int Jy = (g.k - ry + s - 1) / s, Jx = (g.k - rx + s - 1) / s;
                const bool active = Jy > 0 && Jx > 0;
                if (active != (pass == 0)) continue;
                p.cls_ry[k] = ry;
                p.cls_rx[k] = rx;
                p.cls_t0[k] = ntap;
                p.cls_nt[k] = active ? Jy * Jx : 0;
                if (active)
                    for (int jy = 0; jy < Jy; ++jy)
                        for (int jx = 0; jx < Jx; ++jx) {
                            if (ntap >= MAX_TAPS) return false;
                            p.tap_shift[ntap] = (p.gy - jy) * p.P + (p.gx - jx);
                            p.tap_w[ntap] = (ry + s * jy) * g.k + (rx + s * jx);
                            ntap++;
                        }
                k++;
            }
    p.nact = 0;
    for (int i = 0; i < p.ncls; ++i) p.nact += p.cls_nt[i] > 0;
    if (p.nact == 0) return false;
    const int max_shift = p.gy * p.P + p.gx;
    p.items = 2 * wa.hh * wa.hw;
    int vt = (p.items + 31) / 32;
    p.wpi = vt >= 8 ? 8 : (vt >= 4 ? 4 : (vt >= 2 ? 2 : 1));
    p.w_stage_bytes = g.k * g.k * p.Np * 32;
    const int w_all = p.w_stage_bytes * p.nchunk;
    p.w_resident = w_all <= 64 * 1024 ? 1 : 0;
    const int w_bytes = p.w_resident ? w_all : 2 * p.w_stage_bytes;
    // largest group (rows per CTA round) that fits TMEM and shared memory; two accumulator sets if possible
    for (int abuf = 2; abuf >= 1; --abuf) {
        const int cols = (int)TMEM_COLS / abuf;
        for (int G = std::min(MAX_G, (int)(cols / p.Np) * BM / std::max(1, p.npos_img) + 1); G >= 1; --G) {
            const int T = (G * p.npos_img + BM - 1) / BM;
            if (p.nact * T * p.Np > cols) continue;
            const int NPOS = (T * BM + max_shift + 7) / 8 * 8;
            const int a_stage = 2 * 2 * NPOS * 16;  // hi and lo, two 4-channel halves each
            const int rc_bytes = 2 * G * p.wpi * 4;
            const int rt_bytes = 2 * G * (int)sizeof(RowGeo);
            const int cp_bytes = out_mode == OUT_CONCRETIZE ? p.nact * T * BM * 4 : 0;
            const int total = 2 * a_stage + w_bytes + rc_bytes + rt_bytes + 64 + cp_bytes + 1024;
            if (total > SMEM_LIMIT || NPOS * 16 >= (1 << 18)) continue;
            p.G = G;
            p.T = T;
            p.NPOS = NPOS;
            p.abuf = abuf;
            p.acc_cols = cols;
            p.a_stage_bytes = 2 * a_stage;  // both stages
            p.w_off = 2 * a_stage;
            p.rc_off = p.w_off + w_bytes;
            p.rt_off = p.rc_off + (rc_bytes + 15) / 16 * 16;
            p.cp_off = p.rt_off + (rt_bytes + 63) / 64 * 64;
            p.inv_plane = 1.f / (float)(wa.hh * wa.hw);
            p.inv_wa = 1.f / (float)wa.hw;
            p.inv_npos = 1.f / (float)p.npos_img;
            p.inv_p = 1.f / (float)p.P;
            // a group should not leave most of a tile empty when one row already fills several tiles
            return true;
        }
    }
    return false;
}

size_t smem_bytes(const ConvTcParams& p) {
    const size_t cp_bytes = p.out_mode == OUT_CONCRETIZE ? (size_t)p.nact * p.T * BM * 4 : 0;
    return (size_t)p.cp_off + cp_bytes + 1024;
}

}  // namespace

bool conv_back_tc_supported(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode) {
    ConvTcParams p{};
    p.out_mode = out_mode;
    return plan(g, wa, wd, out_mode, &p);
}

bool conv_back_tc_covers(const ConvGeom& g, const Win& wa, const Win& wd) {
    // a STORE fills every entry of the destination window only when, for every row, the natural window of
    // the rows (the receptive field of wa) covers wd: same origin slopes and an origin offset that puts wd
    // inside it
    if (wd.ay != g.stride * wa.ay || wd.ax != g.stride * wa.ax) return false;
    const int oy = wd.by - (g.stride * wa.by - g.pad), ox = wd.bx - (g.stride * wa.bx - g.pad);
    const int Hn = g.stride * (wa.hh - 1) + g.k, Wn = g.stride * (wa.hw - 1) + g.k;
    return oy >= 0 && ox >= 0 && oy + wd.hh <= Hn && ox + wd.hw <= Wn;
}

cudaError_t launch_conv_back_tc(const RowRef& A, Relax rx, const float* Wtc, const float* bias, long long M,
                                const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                int out_mode, float* out, long long ld_out, float* cst, const float* centres,
                                float eps, int* err, int num_sms, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    ConvTcParams p{};
    p.out_mode = out_mode;
    if (!plan(g, wa, wd, out_mode, &p)) return cudaErrorInvalidValue;
    p.A = A;
    p.rx = rx;
    p.bias = bias;
    p.Wtc = Wtc;
    p.M = M;
    p.g = g;
    p.pg = pg;
    p.ps = ps;
    p.wa = wa;
    p.wd = wd;
    p.out = out;
    p.ld_out = ld_out;
    p.cst = cst;
    p.centres = centres;
    p.eps = eps;
    p.err = err;
    const size_t smem = smem_bytes(p);
    cudaError_t e = allow_dyn_smem((const void*)conv_back_tc, SMEM_LIMIT + 1024);
    if (e != cudaSuccess) return e;
    const long long ngroups = (M + p.G - 1) / p.G;
    const long long grid = std::min<long long>(ngroups, num_sms);
    static const bool trace = getenv("VF_TRACE_CONV_TC") != nullptr;
    if (trace)  // launch plan, for profiling
        fprintf(stderr,
                "conv_back_tc M=%lld ci=%d co=%d k=%d s=%d wa=%dx%d wd=%dx%d mode=%d G=%d T=%d nact=%d npos=%d abuf=%d "
                "smem=%zu groups=%lld\n",
                M, g.ci, g.co, g.k, g.stride, wa.hh, wa.hw, wd.hh, wd.hw, out_mode, p.G, p.T, p.nact, p.npos_img, p.abuf,
                smem, ngroups);
    conv_back_tc<<<(unsigned)grid, NUM_THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace vf
