// CROWN back-substitution through a convolution node (transposed convolution of the rows).
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.2 and §4.2 (bounds through convolutional layers) and §1
// (the linear relaxation matrices A).
//
// For z = conv(h) + b and coefficient rows Lambda over z (length C_out * H_out * W_out):
//   Lambda_h[ci, y, x] = sum_{co, p, q} Lambda[co, (y + pad - p) / s, (x + pad - q) / s] * W[co, ci, p, q]
//   (terms whose source index is fractional or outside the output map are absent)
//   const += sum_{co, i, j} relax(Lambda)[co, i, j] * b[co]  (+ the relaxation intercepts)
//
// Work item = (8 rows, one spatial tile of the input map). Per chunk of output channels the CTA stages
// the weights [cc][k][k][ci4] and the relaxed window of Lambda the tile reads, laid out
// [cc][wy][wx][8 rows] so that one pair of 128-bit loads gives a tap's value for all 8 rows; warp w
// stages row w (lanes along the window's columns, so global reads are contiguous). Threads own one input
// pixel x 4 input channels x 8 rows (32 accumulators); pixels are ordered by their position modulo the
// stride, so all threads of a warp share the same valid kernel taps.
//
// Row constants: every output pixel is owned by exactly one tile (the tile holding input pixel
// (s*oy, s*ox)); while staging, each tile adds the relaxation intercept and bias terms of the pixels it
// owns to a per-tile partial, cpart[tile * M + m]. For the node that reads the input the concretised
// outputs are added to the same partial. The partials are summed later in a fixed order, so results are
// bitwise reproducible.
#include <algorithm>

#include "vf_internal.cuh"

namespace vf {

namespace {

constexpr int kThreads = 256;
constexpr int RG = 8;  // rows per work item == warps per CTA

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }
__device__ __forceinline__ int ceil_div(int a, int b) { return -floor_div(-a, b); }

struct ConvTiling {
    int th, tw, ntx, nty;  // input tile and tile grid
    int ncg;               // groups of 4 input channels
    int cc;                // output channels per staged chunk
    int wh_max, ww_max;    // largest Lambda window a tile reads
};

__global__ void __launch_bounds__(kThreads, 2)
conv_back_ffma(RowRef A, Relax rx, const float* __restrict__ W, const float* __restrict__ bias, long long M, ConvGeom g,
               PassGeom pg, int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cpart,
               const float* __restrict__ centres, float eps, ConvTiling t) {
    extern __shared__ float4 smem4[];
    __shared__ float red[RG][kThreads / 32];
    __shared__ const float* rowp[RG];  // this item's row addresses (null past the end)
    __shared__ long long rowb[RG];     // and their centres
    float* sm = reinterpret_cast<float*>(smem4);
    const int ci4 = t.ncg * 4;
    const int kk = g.k * g.k;
    float* Ws = sm;                    // [cc][p][q][ci4]
    float* Ls = sm + t.cc * kk * ci4;  // [cc][wy][wx][RG]
    // relaxation window shared by the item's rows, and per-thread constant accumulators [RG][threads]
    float4* Ps = reinterpret_cast<float4*>(Ls + (size_t)t.cc * RG * t.wh_max * t.ww_max);
    const size_t lsps = (size_t)t.cc * t.wh_max * t.ww_max * (RG + 4);
    const size_t trs = (size_t)RG * t.ncg * 4 * t.th * t.tw;
    float* cst_s = Ls + (lsps > trs ? lsps : trs);  // after everything the store transpose may overwrite
    const int hw_o = g.ho * g.wo;
    const int nOut = g.co * hw_o;
    const int S = g.h * g.w;
    const long long nIn = (long long)g.ci * S;
    const int ntiles = t.ntx * t.nty;
    const long long items = ((M + RG - 1) / RG) * ntiles;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int st = g.stride;
    // thread -> (parity class, pixel within class, channel group), channel group fastest
    const int npc = (t.th / st) * (t.tw / st);  // pixels per parity class
    const int cg = tid % t.ncg;
    const int rest = tid / t.ncg;
    const int cls = rest / npc, lp = rest % npc;
    const int py = cls / st, px = cls % st;
    const int yy = lp / (t.tw / st), xx = lp % (t.tw / st);
    const bool thread_used = cls < st * st;
    const bool w_once = g.co <= t.cc;  // one chunk covers all output channels: stage W once per CTA

    if (w_once) {
        for (int e = tid; e < g.co * kk * ci4; e += kThreads) {
            const int ci = e % ci4;
            const int r2 = e / ci4;
            const int q = r2 % g.k, p = (r2 / g.k) % g.k, c = r2 / kk;
            Ws[e] = (ci < g.ci) ? W[(((long long)c * g.ci + ci) * g.k + p) * g.k + q] : 0.f;
        }
    }

    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const long long m0 = (it / ntiles) * RG;
        const int tile = (int)(it % ntiles);
        const int y0 = (tile / t.ntx) * t.th, x0 = (tile % t.ntx) * t.tw;
        // output rows/cols that contribute to input rows y0 .. y0 + th - 1 (and columns likewise)
        const int oy_lo = max(0, ceil_div(y0 + g.pad - (g.k - 1), st));
        const int oy_hi = min(g.ho - 1, floor_div(y0 + t.th - 1 + g.pad, st));
        const int ox_lo = max(0, ceil_div(x0 + g.pad - (g.k - 1), st));
        const int ox_hi = min(g.wo - 1, floor_div(x0 + t.tw - 1 + g.pad, st));
        const int wh = max(0, oy_hi - oy_lo + 1), ww = max(0, ox_hi - ox_lo + 1);
        const int y = y0 + yy * st + py, x = x0 + xx * st + px;
        const bool active = thread_used && y < g.h && x < g.w;

        float acc[RG][4];
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][i] = 0.f;
        __syncthreads();  // rowp/rowb of the previous item are no longer read
        if (tid < RG) {
            const long long m = m0 + tid;
            rowp[tid] = (m < M) ? A.row(m) : nullptr;
            rowb[tid] = (m < M) ? (pg.pass_m0 + m) / pg.R_pass : 0;
        }
#pragma unroll
        for (int r = 0; r < RG; ++r) cst_s[r * kThreads + tid] = 0.f;

        for (int c0 = 0; c0 < g.co; c0 += t.cc) {
            const int cc = min(t.cc, g.co - c0);
            __syncthreads();  // the previous chunk is no longer read
            if (!w_once) {
                for (int e = tid; e < cc * kk * ci4; e += kThreads) {
                    const int ci = e % ci4;
                    const int r2 = e / ci4;
                    const int q = r2 % g.k, p = (r2 / g.k) % g.k, c = r2 / kk;
                    Ws[e] = (ci < g.ci) ? W[(((long long)(c0 + c) * g.ci + ci) * g.k + p) * g.k + q] : 0.f;
                }
            }
            {
                // All 256 threads stage: first (if the item's rows share one centre) the relaxation
                // window once, then the 8 rows' Lambda windows, relaxed, with the owned-pixel constants.
                // Element indices are split with float reciprocals (exact for these small sizes).
                const int nwin = cc * wh * ww;
                const float inv_ww = 1.f / (float)ww, inv_wh = 1.f / (float)wh;
                // the item's valid rows are consecutive, so they share a centre iff the first and the last
                // valid row do (rows past M are padding and carry no centre)
                const int nvalid = (int)((M - m0) < RG ? (M - m0) : RG);
                const bool shared_p = (rx.P != nullptr) && rowb[0] == rowb[nvalid - 1];
                if (shared_p) {
                    const float4* P0 = rx.P + rowb[0] * nOut;
                    for (int e = tid; e < nwin; e += kThreads) {
                        const int t1 = (int)(((float)e + 0.5f) * inv_ww);
                        const int wx = e - t1 * ww;
                        const int c = (int)(((float)t1 + 0.5f) * inv_wh);
                        const int wy = t1 - c * wh;
                        Ps[e] = P0[(c0 + c) * hw_o + (oy_lo + wy) * g.wo + (ox_lo + wx)];
                    }
                    __syncthreads();
                }
                // lanes = 8 rows x 4 consecutive window positions: the interleaved [pos][row] smem
                // stores of a warp are 32 consecutive floats (no bank conflicts)
                const int r = lane & (RG - 1);
                const float* rp = rowp[r];
                const float4* Pr = (rx.P != nullptr && !shared_p && rp != nullptr) ? rx.P + rowb[r] * nOut : nullptr;
                float* cacc = cst_s + r * kThreads + tid;
                constexpr int NB = 4;  // window positions per batch and thread: loads first, then use
                const int step = 4 * (kThreads / 32);
                for (int pb0 = warp * 4; pb0 < nwin; pb0 += NB * step) {
                    float xv[NB];
                    float4 pr[NB];
                    int jj[NB];
#pragma unroll
                    for (int u = 0; u < NB; ++u) {
                        const int ew = pb0 + u * step + (lane >> 3);
                        jj[u] = -1;
                        xv[u] = 0.f;
                        if (ew < nwin && rp != nullptr) {
                            const int t1 = (int)(((float)ew + 0.5f) * inv_ww);
                            const int wx = ew - t1 * ww;
                            const int c = (int)(((float)t1 + 0.5f) * inv_wh);
                            const int wy = t1 - c * wh;
                            const int j = (c0 + c) * hw_o + (oy_lo + wy) * g.wo + (ox_lo + wx);
                            jj[u] = j;
                            xv[u] = rp[j];
                            if (rx.P != nullptr) pr[u] = shared_p ? Ps[ew] : Pr[j];
                        }
                    }
#pragma unroll
                    for (int u = 0; u < NB; ++u) {
                        const int ew = pb0 + u * step + (lane >> 3);
                        if (ew >= nwin) break;
                        float v = 0.f;
                        if (jj[u] >= 0) {
                            v = xv[u];
                            float tcst = 0.f;
                            if (rx.P != nullptr) {
                                v = (xv[u] >= 0.f) ? xv[u] * pr[u].x : xv[u] * pr[u].y;
                                if (rx.count_const) tcst = fminf(xv[u], 0.f) * pr[u].z;
                            }
                            const int j = jj[u];
                            const int cch = j / hw_o;  // absolute output channel
                            const int oy = (j - cch * hw_o) / g.wo, ox = j - cch * hw_o - oy * g.wo;
                            // the tile owns output pixel (oy, ox) iff it holds input pixel (s*oy, s*ox), clamped
                            const bool own = (min(oy * st, g.h - 1) >= y0) && (min(oy * st, g.h - 1) <= y0 + t.th - 1) &&
                                             (min(ox * st, g.w - 1) >= x0) && (min(ox * st, g.w - 1) <= x0 + t.tw - 1);
                            if (cpart != nullptr && own) *cacc += tcst + (bias != nullptr ? v * bias[cch] : 0.f);
                        }
                        Ls[ew * RG + r] = v;  // [c][wy][wx][r]
                    }
                }
            }
            __syncthreads();
            if (active) {
                for (int p = 0; p < g.k; ++p) {
                    const int ty = y + g.pad - p;
                    if (ty < 0 || (ty % st) != 0) continue;
                    const int oy = ty / st;
                    if (oy < oy_lo || oy > oy_hi) continue;
                    for (int q = 0; q < g.k; ++q) {
                        const int tx = x + g.pad - q;
                        if (tx < 0 || (tx % st) != 0) continue;
                        const int ox = tx / st;
                        if (ox < ox_lo || ox > ox_hi) continue;
                        const float* lp = Ls + ((oy - oy_lo) * ww + (ox - ox_lo)) * RG;
                        const float* wp = Ws + (((w_once ? c0 : 0) * g.k + p) * g.k + q) * ci4 + cg * 4;
                        const int lstride = wh * ww * RG, wstride = kk * ci4;
                        for (int c = 0; c < cc; ++c) {
                            const float4 w4 = *reinterpret_cast<const float4*>(wp + c * wstride);
                            const float4 la = *reinterpret_cast<const float4*>(lp + c * lstride);
                            const float4 lb = *reinterpret_cast<const float4*>(lp + c * lstride + 4);
                            const float lv[RG] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
                            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int r = 0; r < RG; ++r)
#pragma unroll
                                for (int i = 0; i < 4; ++i) acc[r][i] = fmaf(lv[r], wv[i], acc[r][i]);
                        }
                    }
                }
            }
        }

        // per-row partial of this tile: constants owned by the tile (+ concretised outputs at the input)
        float conc[RG];
#pragma unroll
        for (int r = 0; r < RG; ++r) conc[r] = 0.f;
        if (out_mode == OUT_CONCRETIZE) {
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                if (active && rowp[r] != nullptr) {
                    const float* c = centres + rowb[r] * nIn;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int ci = cg * 4 + i;
                        if (ci < g.ci) conc[r] += fmaf(acc[r][i], c[(long long)ci * S + y * g.w + x], -eps * fabsf(acc[r][i]));
                    }
                }
            }
        } else {
            // transpose through smem (over the Lambda staging area) so that global stores run along x
            float* T = Ls;  // [RG][ci4][th * tw]
            const int tp = t.th * t.tw;
            __syncthreads();  // every thread is done reading Ls
            if (active) {
                const int pl = (y - y0) * t.tw + (x - x0);
#pragma unroll
                for (int r = 0; r < RG; ++r)
#pragma unroll
                    for (int i = 0; i < 4; ++i) T[(r * ci4 + cg * 4 + i) * tp + pl] = acc[r][i];
            }
            __syncthreads();
            const int ntot = RG * g.ci * tp;
            const int lg_tp = 31 - __clz(tp);  // tp = th * tw is a power of two
            const float inv_ci = 1.f / (float)g.ci;
            constexpr int NB = 4;
            for (int e0 = tid; e0 < ntot; e0 += NB * kThreads) {
                float* op[NB];
                float val[NB], old[NB];
#pragma unroll
                for (int u = 0; u < NB; ++u) {
                    const int e = e0 + u * kThreads;
                    op[u] = nullptr;
                    if (e >= ntot) continue;
                    const int pl = e & (tp - 1);
                    const int rest2 = e >> lg_tp;
                    const int r = (int)(((float)rest2 + 0.5f) * inv_ci);
                    const int ci = rest2 - r * g.ci;
                    const int yy2 = y0 + (pl / t.tw), xx2 = x0 + (pl % t.tw);
                    if (m0 + r >= M || yy2 >= g.h || xx2 >= g.w) continue;
                    op[u] = out + (m0 + r) * ld_out + (long long)ci * S + yy2 * g.w + xx2;
                    val[u] = T[(r * ci4 + ci) * tp + pl];
                    old[u] = (out_mode == OUT_ACCUM) ? *op[u] : 0.f;
                }
#pragma unroll
                for (int u = 0; u < NB; ++u)
                    if (op[u] != nullptr) *op[u] = old[u] + val[u];
            }
        }
        if (cpart != nullptr) {
            // warp w contributes conc[0..7] (all rows) and cs (row w); reduce over the block, fixed order
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                float v = conc[r] + cst_s[r * kThreads + tid];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) red[r][warp] = v;
            }
            __syncthreads();
            if (tid < RG && m0 + tid < M) {
                float s = 0.f;
                for (int w = 0; w < kThreads / 32; ++w) s += red[tid][w];
                cpart[(long long)tile * M + m0 + tid] = s;
            }
        }
    }
}

ConvTiling make_tiling(const ConvGeom& g) {
    ConvTiling t;
    t.ncg = (g.ci + 3) / 4;
    if (t.ncg > 2 && t.ncg < 4) t.ncg = 4;  // keep ncg a power of two so pixel tiles are rectangles
    if (t.ncg > 4 && t.ncg < 8) t.ncg = 8;
    if (t.ncg > 8 && t.ncg < 16) t.ncg = 16;
    const int npix = std::max(1, kThreads / t.ncg);
    // tile width/height: powers of two, multiples of the stride, covering npix pixels
    int tw = 1;
    while (tw * tw < npix) tw *= 2;
    int th = npix / tw;
    tw = std::max(tw, g.stride);
    th = std::max(th, g.stride);
    // shrink a tile that overhangs a small map (still a multiple of the stride)
    while (tw > g.stride && tw / 2 >= g.w) tw /= 2;
    while (th > g.stride && th / 2 >= g.h) th /= 2;
    t.tw = tw;
    t.th = th;
    t.ntx = (g.w + t.tw - 1) / t.tw;
    t.nty = (g.h + t.th - 1) / t.th;
    t.wh_max = (t.th - 1 + g.k - 1) / g.stride + 2;
    t.ww_max = (t.tw - 1 + g.k - 1) / g.stride + 2;
    t.cc = std::min(g.co, 64);
    // keep the staged chunk within ~96 KB so that two CTAs fit on an SM
    while (t.cc > 1 && (size_t)t.cc * (g.k * g.k * t.ncg * 4 + (RG + 4) * t.wh_max * t.ww_max) * 4 > 90 * 1024) t.cc /= 2;
    return t;
}

}  // namespace

size_t conv_back_smem_bytes(const ConvGeom& g) {
    const ConvTiling t = make_tiling(g);
    const size_t ws = (size_t)t.cc * g.k * g.k * t.ncg * 4;
    const size_t ls = (size_t)t.cc * RG * t.wh_max * t.ww_max;
    const size_t tr = (size_t)RG * t.ncg * 4 * t.th * t.tw;  // store transpose, aliased over Ls (and Ps)
    const size_t ps = (size_t)t.cc * t.wh_max * t.ww_max * 4;  // float4 relaxation window
    const size_t cs = (size_t)RG * kThreads;                     // per-thread constant accumulators
    return (ws + std::max(ls + ps, tr) + cs) * sizeof(float);
}

int conv_back_tiles(const ConvGeom& g) {
    const ConvTiling t = make_tiling(g);
    return t.ntx * t.nty;
}

bool conv_back_supported(const ConvGeom& g) {
    // strides 1, 2 or 4 (tiles are powers of two); the tile that owns output pixel (oy, ox) must read it,
    // which needs pad <= k - 1 and s * (H_out - 1) <= H - 1 + pad (likewise for the width)
    return (g.stride == 1 || g.stride == 2 || g.stride == 4) && g.pad <= g.k - 1 &&
           g.stride * (g.ho - 1) <= g.h - 1 + g.pad && g.stride * (g.wo - 1) <= g.w - 1 + g.pad &&
           conv_back_smem_bytes(g) <= 200 * 1024;
}

cudaError_t launch_conv_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M,
                             const ConvGeom& g, PassGeom pg, int out_mode, float* out, long long ld_out, float* cpart,
                             const float* centres, float eps, int num_sms, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    const ConvTiling t = make_tiling(g);
    const size_t smem = conv_back_smem_bytes(g);
    cudaError_t e = allow_dyn_smem((const void*)conv_back_ffma, 200 * 1024);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv_back_ffma, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const long long items = ((M + RG - 1) / RG) * (long long)(t.ntx * t.nty);
    long long grid = (long long)num_sms * per_sm;
    if (grid > items) grid = items;
    conv_back_ffma<<<(unsigned)grid, kThreads, smem, s>>>(A, rx, W, bias, M, g, pg, out_mode, out, ld_out, cpart,
                                                          centres, eps, t);
    return cudaGetLastError();
}

}  // namespace vf
