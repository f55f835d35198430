// Receptive-field windows for the rows of intermediate passes that start at a convolution.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 and §4.1 (the linear relaxation matrices A dominate the memory and
// grow with the layer width) and §2.1 (CROWN bounds for every intermediate ReLU layer).
//
// The pass over node p starts from one row per neuron j = (c_j, y_j, x_j) of p and its negation. Going
// back through convolutions the row is nonzero only inside the receptive field of (y_j, x_j), a window
// whose origin is affine in (y_j, x_j) and whose size is the same for every row of the pass. Each
// nonzero entry gets the same products and terms as in the whole-map computation; entries outside the
// window are zero there and are not stored here.
#include <algorithm>

#include "vf_internal.cuh"

namespace vf {

namespace {

struct StartPos {
    int yj, xj, cj;
    float sg;
    long long b;  // centre
};

__device__ __forceinline__ StartPos start_pos(const PassStart& ps, const PassGeom& pg, long long m) {
    const long long g = pg.pass_m0 + m;
    const long long r = g % pg.R_pass;
    const long long j = r % ps.n;
    StartPos s;
    s.sg = (r < ps.n) ? 1.f : -1.f;
    s.xj = (int)(j % ps.w);
    s.yj = (int)((j / ps.w) % ps.h);
    s.cj = (int)(j / ((long long)ps.h * ps.w));
    s.b = g / pg.R_pass;
    return s;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

unsigned warp_rows_grid(long long M, int rows_per_cta, int ctas_per_sm) {
    long long g = (M + rows_per_cta - 1) / rows_per_cta;
    const long long cap = 148LL * ctas_per_sm;
    if (g > cap) g = cap;
    return (unsigned)(g < 1 ? 1 : g);
}

// Start rows: +-W[c_j, :, p, q] at input position (s*y_j - pad + p, s*x_j - pad + q). One warp per row.
__global__ void __launch_bounds__(256)
conv_start_rows_win_k(float* __restrict__ out, long long ld, long long M, PassGeom pg, PassStart ps,
                      const float* __restrict__ W, ConvGeom g, Win wd, int accumulate) {
    const int nwin = wd.C * wd.hh * wd.hw;
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const StartPos sp = start_pos(ps, pg, m);
        const int oy = wd.ay * sp.yj + wd.by, ox = wd.ax * sp.xj + wd.bx;
        const int fy = sp.yj * g.stride - g.pad, fx = sp.xj * g.stride - g.pad;
        float* o = out + m * ld;
        for (int e = lane; e < nwin; e += 32) {
            const int dx = e % wd.hw, dy = (e / wd.hw) % wd.hh, ci = e / (wd.hw * wd.hh);
            const int y = oy + dy, x = ox + dx;
            const int p = y - fy, q = x - fx;
            float v = 0.f;
            if (y >= 0 && y < g.h && x >= 0 && x < g.w && p >= 0 && p < g.k && q >= 0 && q < g.k)
                v = sp.sg * W[(((long long)sp.cj * g.ci + ci) * g.k + p) * g.k + q];
            o[e] = accumulate ? o[e] + v : v;
        }
    }
}

// Identity start rows (+-e_j) in window `wd` of the start node's map (the identity shortcut of a pass that
// starts at a residual add). One warp per row.
__global__ void __launch_bounds__(256)
ident_rows_win_k(float* __restrict__ out, long long ld, long long M, PassGeom pg, PassStart ps, Win wd,
                 int accumulate) {
    const int nwin = wd.C * wd.hh * wd.hw;
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const StartPos sp = start_pos(ps, pg, m);
        const int dy = sp.yj - (wd.ay * sp.yj + wd.by), dx = sp.xj - (wd.ax * sp.xj + wd.bx);
        const int hit = (sp.cj * wd.hh + dy) * wd.hw + dx;  // inside the window by construction
        float* o = out + m * ld;
        if (accumulate) {
            if (lane == 0) o[hit] += sp.sg;
        } else {
            for (int e = lane; e < nwin; e += 32) o[e] = (e == hit) ? sp.sg : 0.f;
        }
    }
}

// Transposed convolution on windowed rows. One warp per row, `nwarps` rows per CTA. The relaxed row
// window over the conv output is staged in shared memory ([co][hh][hw], zeros off the map); each lane
// then owns output positions of the destination window and CB input channels at a time, gathering its
// (k/s)^2 taps x co products. Wt is [k*k][tap_stride] with tap (p, q) holding [co][ci_pad].
template <int CB>
__global__ void __launch_bounds__(256)
conv_back_win_k(RowRef A, Relax rx, const float* __restrict__ Wt, int tap_stride, int ci_pad, int w_in_smem,
                const float* __restrict__ bias, long long M, ConvGeom g, PassGeom pg, PassStart ps, Win wa, Win wd,
                int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cst,
                const float* __restrict__ centres, float eps, int nwarps, int stage_floats) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    const int kk = g.k * g.k;
    const int nW = w_in_smem ? kk * tap_stride : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (w_in_smem) {
        const float4* src = reinterpret_cast<const float4*>(Wt);
        for (int e = threadIdx.x; e < nW / 4; e += blockDim.x) smem4[e] = src[e];
    }
    __syncthreads();
    if (warp >= nwarps) return;
    const float* Ws = w_in_smem ? sm : Wt;
    float* As = sm + nW + warp * stage_floats;
    const int hw_o = g.ho * g.wo;
    const long long nOut = (long long)g.co * hw_o;
    const int astr = wa.hh * wa.hw;
    const int na = wa.C * astr;
    const int npos = wd.hh * wd.hw;
    const int nchunks = ci_pad / CB;
    const int items = npos * nchunks;
    const int KS = (g.k + g.stride - 1) / g.stride;
    const long long S = (long long)g.h * g.w;
    for (long long m = (long long)blockIdx.x * nwarps + warp; m < M; m += (long long)gridDim.x * nwarps) {
        const StartPos sp = start_pos(ps, pg, m);
        const int aoy = wa.ay * sp.yj + wa.by, aox = wa.ax * sp.xj + wa.bx;
        const int doy = wd.ay * sp.yj + wd.by, dox = wd.ax * sp.xj + wd.bx;
        const float* arow = A.row(m);
        float cs = 0.f;
        for (int e = lane; e < na; e += 32) {
            const int dx = e % wa.hw, dy = (e / wa.hw) % wa.hh, co = e / astr;
            const int y = aoy + dy, x = aox + dx;
            float v = 0.f;
            if (y >= 0 && y < g.ho && x >= 0 && x < g.wo) {
                const float xv = arow[e];
                v = xv;
                if (rx.P != nullptr) {
                    const float4 pr = rx.P[sp.b * nOut + (long long)co * hw_o + y * g.wo + x];
                    v = (xv >= 0.f) ? xv * pr.x : xv * pr.y;
                    if (rx.count_const) cs = fmaf(fminf(xv, 0.f), pr.z, cs);
                }
                if (bias != nullptr) cs = fmaf(v, bias[co], cs);
            }
            As[e] = v;
        }
        __syncwarp();
        // receptive field of the staged window on the input map (positions outside get no taps)
        const int fy0 = g.stride * aoy - g.pad, fy1 = g.stride * (aoy + wa.hh - 1) - g.pad + g.k;
        const int fx0 = g.stride * aox - g.pad, fx1 = g.stride * (aox + wa.hw - 1) - g.pad + g.k;
        const float* crow = (out_mode == OUT_CONCRETIZE) ? centres + sp.b * (long long)g.ci * S : nullptr;
        float* orow = (out_mode == OUT_CONCRETIZE) ? nullptr : out + m * ld_out;
        float conc = 0.f;
        for (int it = lane; it < items; it += 32) {
            const int chunk = it / npos, pos = it - chunk * npos;
            const int dy = pos / wd.hw, dx = pos - dy * wd.hw;
            const int Y = doy + dy, X = dox + dx;
            float acc[CB];
#pragma unroll
            for (int i = 0; i < CB; ++i) acc[i] = 0.f;
            const bool live = Y >= 0 && Y < g.h && X >= 0 && X < g.w && Y >= fy0 && Y < fy1 && X >= fx0 && X < fx1;
            if (live) {
                const int ry = Y + g.pad, rxx = X + g.pad;
                const int p0 = ry % g.stride, q0 = rxx % g.stride;
                const int oy0 = ry / g.stride - aoy, ox0 = rxx / g.stride - aox;  // window row/col of tap p0/q0
                for (int tp = 0; tp < KS; ++tp) {
                    const int p = p0 + g.stride * tp, ay = oy0 - tp;
                    if (p >= g.k || ay < 0 || ay >= wa.hh) continue;
                    for (int tq = 0; tq < KS; ++tq) {
                        const int q = q0 + g.stride * tq, ax = ox0 - tq;
                        if (q >= g.k || ax < 0 || ax >= wa.hw) continue;
                        const float* ap = As + ay * wa.hw + ax;
                        const float4* wp =
                            reinterpret_cast<const float4*>(Ws + (p * g.k + q) * tap_stride + chunk * CB);
                        for (int co = 0; co < g.co; ++co) {
                            const float a = ap[co * astr];
#pragma unroll
                            for (int i = 0; i < CB / 4; ++i) {
                                const float4 w4 = wp[co * (ci_pad / 4) + i];
                                acc[4 * i + 0] = fmaf(a, w4.x, acc[4 * i + 0]);
                                acc[4 * i + 1] = fmaf(a, w4.y, acc[4 * i + 1]);
                                acc[4 * i + 2] = fmaf(a, w4.z, acc[4 * i + 2]);
                                acc[4 * i + 3] = fmaf(a, w4.w, acc[4 * i + 3]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < CB; ++i) {
                const int ci = chunk * CB + i;
                if (ci >= g.ci) break;
                if (crow != nullptr) {
                    if (live) conc += fmaf(acc[i], crow[ci * S + (long long)Y * g.w + X], -eps * fabsf(acc[i]));
                } else {
                    float* o = orow + (long long)ci * npos + pos;
                    *o = (out_mode == OUT_ACCUM) ? *o + acc[i] : acc[i];
                }
            }
        }
        const float tot = warp_sum(cs + conc);
        if (lane == 0 && cst != nullptr) cst[m] += tot;
        __syncwarp();  // the next row overwrites this warp's staging
    }
}

// out (=, +=) relax(A) moved from window wa into window wd of the same C x H x W map. One warp per row.
__global__ void __launch_bounds__(256)
rewin_rows_k(RowRef A, Relax rx, long long M, int C, int H, int Wd, PassGeom pg, PassStart ps, Win wa, Win wd,
             float* __restrict__ out, long long ld_out, int accumulate, float* __restrict__ cst) {
    const int lane = threadIdx.x & 31;
    const long long n = (long long)C * H * Wd;
    const int nd = wd.C * wd.hh * wd.hw;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const StartPos sp = start_pos(ps, pg, m);
        const int aoy = wa.ay * sp.yj + wa.by, aox = wa.ax * sp.xj + wa.bx;
        const int doy = wd.ay * sp.yj + wd.by, dox = wd.ax * sp.xj + wd.bx;
        const float* a = A.row(m);
        float* o = out + m * ld_out;
        float cs = 0.f;
        for (int e = lane; e < nd; e += 32) {
            const int dx = e % wd.hw, dy = (e / wd.hw) % wd.hh, c = e / (wd.hw * wd.hh);
            const int Y = doy + dy, X = dox + dx;
            const int ry = Y - aoy, rxx = X - aox;
            float r = 0.f;
            if (Y >= 0 && Y < H && X >= 0 && X < Wd && ry >= 0 && ry < wa.hh && rxx >= 0 && rxx < wa.hw) {
                const float x = a[((long long)c * wa.hh + ry) * wa.hw + rxx];
                r = x;
                if (rx.P != nullptr) {
                    const float4 p = rx.P[sp.b * n + ((long long)c * H + Y) * Wd + X];
                    r = (x >= 0.f) ? x * p.x : x * p.y;
                    if (rx.count_const) cs = fmaf(fminf(x, 0.f), p.z, cs);
                }
            }
            o[e] = accumulate ? o[e] + r : r;
        }
        if (rx.P != nullptr && rx.count_const && cst != nullptr) {
            const float t = warp_sum(cs);
            if (lane == 0) cst[m] += t;
        }
    }
}

template <int CB>
cudaError_t launch_back_cb(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                           const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd, int out_mode,
                           float* out, long long ld_out, float* cst, const float* centres, float eps,
                           const WinLaunch& L, cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(conv_back_win_k<CB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kWinSmemLimit);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    conv_back_win_k<CB><<<warp_rows_grid(M, L.nwarps, L.ctas_per_sm), 32 * L.nwarps, L.smem, s>>>(
        A, rx, ww.Wt, ww.tap_stride, ww.ci_pad, L.w_in_smem, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
        centres, eps, L.nwarps, L.stage_floats);
    return cudaGetLastError();
}

}  // namespace

int win_ci_block(int ci) { return ci <= 4 ? 4 : (ci <= 8 ? 8 : 16); }

bool conv_back_win_plan(const ConvGeom& g, const WinWeights& ww, const Win& wa, WinLaunch* L) {
    const size_t wbytes = (size_t)g.k * g.k * ww.tap_stride * sizeof(float);
    L->stage_floats = (wa.C * wa.hh * wa.hw + 3) / 4 * 4;
    const size_t stage = (size_t)L->stage_floats * sizeof(float);
    if (stage > (size_t)kWinSmemLimit) return false;
    int nw = (int)std::min<size_t>(8, ((size_t)kWinSmemLimit - std::min(wbytes, (size_t)kWinSmemLimit)) / stage);
    if (wbytes <= (size_t)kWinSmemLimit && nw >= 4) {
        L->w_in_smem = 1;
    } else {
        L->w_in_smem = 0;
        nw = (int)std::min<size_t>(8, (size_t)kWinSmemLimit / stage);
        if (nw < 1) return false;
    }
    L->nwarps = nw;
    L->smem = (L->w_in_smem ? wbytes : 0) + (size_t)nw * stage;
    // CTAs resident per SM by shared memory (228 KB per SM, 1 KB reserved per CTA), at most 8
    int per_sm = (int)(233472 / (L->smem + 1024));
    L->ctas_per_sm = std::max(1, std::min(8, per_sm));
    return true;
}

cudaError_t launch_conv_start_rows_win(float* out, long long ld, long long M, PassGeom pg, PassStart ps, const float* W,
                                       const ConvGeom& g, const Win& wd, int accumulate, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    conv_start_rows_win_k<<<warp_rows_grid(M, 8, 8), 256, 0, s>>>(out, ld, M, pg, ps, W, g, wd, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_conv_back_win(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                                 const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                 int out_mode, float* out, long long ld_out, float* cst, const float* centres, float eps,
                                 cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    WinLaunch L;
    if (!conv_back_win_plan(g, ww, wa, &L)) return cudaErrorInvalidConfiguration;
    switch (ww.cb) {
        case 4:
            return launch_back_cb<4>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres, eps, L, s);
        case 8:
            return launch_back_cb<8>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres, eps, L, s);
        default:
            return launch_back_cb<16>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres, eps, L,
                                      s);
    }
}

cudaError_t launch_ident_rows_win(float* out, long long ld, long long M, PassGeom pg, PassStart ps, const Win& wd,
                                  int accumulate, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    ident_rows_win_k<<<warp_rows_grid(M, 8, 8), 256, 0, s>>>(out, ld, M, pg, ps, wd, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_rewin_rows(const RowRef& A, Relax rx, long long M, int C, int H, int W, PassGeom pg, PassStart ps,
                              const Win& wa, const Win& wd, float* out, long long ld_out, int accumulate, float* cst,
                              cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    rewin_rows_k<<<warp_rows_grid(M, 8, 8), 256, 0, s>>>(A, rx, M, C, H, W, pg, ps, wa, wd, out, ld_out, accumulate,
                                                          cst);
    return cudaGetLastError();
}

}  // namespace vf
