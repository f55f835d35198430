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
    StartPos s;
    const long long j = start_neuron(pg, ps.n, m, &s.sg);
    s.xj = (int)(j % ps.w);
    s.yj = (int)((j / ps.w) % ps.h);
    s.cj = (int)(j / ((long long)ps.h * ps.w));
    s.b = g / pg.R_pass;
    return s;
}

// n / d for 0 <= n < 2^22 and small d, exact: (n + 0.5) / d is at least 1/(2d) from an integer
__device__ __forceinline__ int fdiv(int n, float inv) { return __float2int_rz(((float)n + 0.5f) * inv); }

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
    const int plane = wd.hh * wd.hw;
    const float inv_plane = 1.f / (float)plane, inv_hw = 1.f / (float)wd.hw;
    const int lane = threadIdx.x & 31;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const StartPos sp = start_pos(ps, pg, m);
        const int oy = wd.ay * sp.yj + wd.by, ox = wd.ax * sp.xj + wd.bx;
        const int fy = sp.yj * g.stride - g.pad, fx = sp.xj * g.stride - g.pad;
        float* o = out + m * ld;
        for (int e = lane; e < nwin; e += 32) {
            const int ci = fdiv(e, inv_plane);
            const int r2 = e - ci * plane;
            const int dy = fdiv(r2, inv_hw), dx = r2 - dy * wd.hw;
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
    const float inv_hw = 1.f / (float)wd.hw, inv_hh = 1.f / (float)wd.hh;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += (long long)gridDim.x * 8) {
        const StartPos sp = start_pos(ps, pg, m);
        const int aoy = wa.ay * sp.yj + wa.by, aox = wa.ax * sp.xj + wa.bx;
        const int doy = wd.ay * sp.yj + wd.by, dox = wd.ax * sp.xj + wd.bx;
        const float* a = A.row(m);
        float* o = out + m * ld_out;
        float cs = 0.f;
        // four entries per lane at a time, every load (coefficient, relaxation, old value) issued before any use
        for (int e0 = lane; e0 < nd; e0 += 128) {
            float x[4], old[4];
            float4 p[4];
            bool in[4], live[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + 32 * u;
                live[u] = e < nd;
                const int q = live[u] ? fdiv(e, inv_hw) : 0, dx = live[u] ? e - q * wd.hw : 0;
                const int c = fdiv(q, inv_hh), dy = q - c * wd.hh;
                const int Y = doy + dy, X = dox + dx;
                const int ry = Y - aoy, rxx = X - aox;
                in[u] = live[u] && Y >= 0 && Y < H && X >= 0 && X < Wd && ry >= 0 && ry < wa.hh && rxx >= 0 &&
                        rxx < wa.hw;
                x[u] = in[u] ? a[((long long)c * wa.hh + ry) * wa.hw + rxx] : 0.f;
                p[u] = (in[u] && rx.P != nullptr) ? rx.P[sp.b * n + ((long long)c * H + Y) * Wd + X]
                                                  : make_float4(1.f, 1.f, 0.f, 0.f);
                old[u] = (live[u] && accumulate) ? o[e] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (!live[u]) continue;
                const float r = (x[u] >= 0.f) ? x[u] * p[u].x : x[u] * p[u].y;
                if (in[u] && rx.P != nullptr && rx.count_const) cs = fmaf(fminf(x[u], 0.f), p[u].z, cs);
                o[e0 + 32 * u] = old[u] + r;
            }
        }
        if (rx.P != nullptr && rx.count_const && cst != nullptr) {
            const float t = warp_sum(cs);
            if (lane == 0) cst[m] += t;
        }
    }
}

// Position-blocked variant of the windowed transposed convolution for stride S and KS = ceil(k / S) taps
// per axis and stride class. The staged row window carries a zero halo, so every tap read stays inside
// the stage and needs no test. Input positions of the receptive field are grouped by stride class
// (y mod S, x mod S); within a class all positions use the same taps. A lane owns PM positions of one
// class (spaced G apart along x, so neighbouring lanes read neighbouring stage words) times CB input
// channels, i.e. PM*CB accumulators that share each staged weight and each staged coefficient.
struct WinClasses {
    int cum[5];  // items before class i (class = pc * S + qc), cum[S*S] = items per row and chunk
    int ny[4], nx[4], G[4];
};


// a[i] for a small runtime i, by selects (keeps the parameter arrays out of local memory)
template <int N>
__device__ __forceinline__ int pick(const int (&a)[N], int i) {
    int v = a[0];
#pragma unroll
    for (int j = 1; j < N; ++j) v = (i == j) ? a[j] : v;
    return v;
}

template <int S, int KS, int CB, int PM>
__global__ void __launch_bounds__(256, 2)
conv_back_win2_k(RowRef A, Relax rx, const float* __restrict__ Wt, int tap_stride, int ci_pad, int w_all,
                 const float* __restrict__ bias, long long M, ConvGeom g, PassGeom pg, PassStart ps, Win wa, Win wd,
                 int out_mode, float* __restrict__ out, long long ld_out, float* __restrict__ cst,
                 const float* __restrict__ centres, float eps, int nwarps, int HH, int HW, int stage_floats,
                 WinClasses cl, float inv_hwd, int zero_fill) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    constexpr int OFF = KS - 1;
    const int kk = g.k * g.k;
    const int slab_ts = g.co * CB + 4;
    const int nW = w_all ? kk * tap_stride : kk * slab_ts;
    const int TSs = w_all ? tap_stride : slab_ts;  // smem stride between taps
    const int COS = w_all ? ci_pad : CB;           // smem stride between output channels
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* As = sm + nW + warp * stage_floats;
    const int HHW = HH * HW;
    const int nst = wa.C * HHW;
    const int hw_o = g.ho * g.wo;
    const long long nOut = (long long)g.co * hw_o;
    const int npos_d = wd.hh * wd.hw;
    const int nchunks = ci_pad / CB;
    const int NYT = S * (wa.hh - 1) + g.k, NXT = S * (wa.hw - 1) + g.k;  // receptive field on the input map
    const long long S_in = (long long)g.h * g.w;
    if (w_all) {
        const float4* src = reinterpret_cast<const float4*>(Wt);
        for (int e = threadIdx.x; e < nW / 4; e += blockDim.x) smem4[e] = src[e];
    }
    // the halo of the stage is zero for every row: clear it once, then rows write the interior only
    for (int e = lane; e < nst; e += 32) As[e] = 0.f;
    const int na = wa.C * wa.hh * wa.hw;
    const float inv_a = 1.f / (float)(wa.hh * wa.hw), inv_aw = 1.f / (float)wa.hw;
    for (long long m0 = (long long)blockIdx.x * nwarps; m0 < M; m0 += (long long)gridDim.x * nwarps) {
        const long long m = m0 + warp;
        const bool active = warp < nwarps && m < M;
        StartPos sp{0, 0, 0, 1.f, 0};
        int aoy = 0, aox = 0, fy0 = 0, fx0 = 0, doy = 0, dox = 0;
        float cs = 0.f, conc = 0.f;
        if (active) {
            sp = start_pos(ps, pg, m);
            aoy = wa.ay * sp.yj + wa.by;
            aox = wa.ax * sp.xj + wa.bx;
            fy0 = S * aoy - g.pad;
            fx0 = S * aox - g.pad;
            doy = wd.ay * sp.yj + wd.by;
            dox = wd.ax * sp.xj + wd.bx;
            const float* arow = A.row(m);
            // four entries per lane at a time: all their loads are issued before any is used
            const float4* Pb = rx.P != nullptr ? rx.P + sp.b * nOut : nullptr;
            for (int e0 = lane; e0 < na; e0 += 128) {
                float xv[4];
                float4 pr[4];
                int co[4], sidx[4];
                bool on[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + 32 * u;
                    const int c = fdiv(e, inv_a);
                    const int r2 = e - c * (wa.hh * wa.hw);
                    const int wy = fdiv(r2, inv_aw);
                    const int wx = r2 - wy * wa.hw;
                    const int y = aoy + wy, x = aox + wx;
                    on[u] = e < na && y >= 0 && y < g.ho && x >= 0 && x < g.wo;
                    co[u] = c;
                    sidx[u] = c * HHW + (wy + OFF) * HW + wx + OFF;
                    xv[u] = on[u] ? arow[e] : 0.f;
                    pr[u] = (on[u] && Pb != nullptr) ? Pb[(long long)c * hw_o + y * g.wo + x] : make_float4(1.f, 1.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (e0 + 32 * u >= na) break;
                    float v = 0.f;
                    if (on[u]) {
                        v = (xv[u] >= 0.f) ? xv[u] * pr[u].x : xv[u] * pr[u].y;
                        if (Pb != nullptr && rx.count_const) cs = fmaf(fminf(xv[u], 0.f), pr[u].z, cs);
                        if (bias != nullptr) cs = fmaf(v, bias[co[u]], cs);
                    }
                    As[sidx[u]] = v;
                }
            }
            if (zero_fill) {  // destination entries outside the receptive field
                float* orow = out + m * ld_out;
                for (int e = lane; e < npos_d; e += 32) {
                    const int yd = fdiv(e, inv_hwd);
                    const int y = doy + yd - fy0, x = dox + (e - yd * wd.hw) - fx0;
                    if (y >= 0 && y < NYT && x >= 0 && x < NXT) continue;
                    for (int ci = 0; ci < g.ci; ++ci) orow[(long long)ci * npos_d + e] = 0.f;
                }
            }
        }
        for (int chunk = 0; chunk < nchunks; ++chunk) {
            if (!w_all) {  // this chunk's weight slab [tap][co][CB]
                __syncthreads();
                for (int e = threadIdx.x; e < kk * g.co * (CB / 4); e += blockDim.x) {
                    const int c4 = e % (CB / 4), rest = e / (CB / 4);
                    const int co = rest % g.co, tap = rest / g.co;
                    smem4[(tap * slab_ts + co * CB) / 4 + c4] =
                        reinterpret_cast<const float4*>(Wt + (size_t)tap * tap_stride + (size_t)co * ci_pad + chunk * CB)[c4];
                }
            }
            __syncthreads();
            if (!active) continue;
            const float* Wc = sm + (w_all ? chunk * CB : 0);
            for (int it = lane; it < cl.cum[S * S]; it += 32) {
                int cls = 0, base = 0;
#pragma unroll
                for (int c2 = 1; c2 < S * S; ++c2)
                    if (it >= cl.cum[c2]) {
                        cls = c2;
                        base = cl.cum[c2];
                    }
                const int pc = cls / S, qc = cls % S;
                const int Gc = pick(cl.G, qc), nxc = pick(cl.nx, qc);
                const int local = it - base;
                const int yq = local / Gc, grp = local - yq * Gc;
                float acc[PM][CB];
#pragma unroll
                for (int i = 0; i < PM; ++i)
#pragma unroll
                    for (int c = 0; c < CB; ++c) acc[i][c] = 0.f;
                bool okp[PM];
#pragma unroll
                for (int i = 0; i < PM; ++i) okp[i] = grp + i * Gc < nxc;
#pragma unroll
                for (int tp = 0; tp < KS; ++tp) {
                    const int p = pc + S * tp;
                    if (p >= g.k) break;
                    const float* arow_s = As + (yq - tp + OFF) * HW + grp;
#pragma unroll
                    for (int tq = 0; tq < KS; ++tq) {
                        const int q = qc + S * tq;
                        if (q >= g.k) break;
                        const float* ab = arow_s + (OFF - tq);
                        const float4* wb = reinterpret_cast<const float4*>(Wc + (p * g.k + q) * TSs);
#pragma unroll 2
                        for (int co = 0; co < g.co; ++co) {
                            float a[PM];
#pragma unroll
                            for (int i = 0; i < PM; ++i) {  // a lane's unused slots read its first (valid) position
                                const float v = ab[co * HHW + (okp[i] ? i * Gc : 0)];
                                a[i] = okp[i] ? v : 0.f;
                            }
#pragma unroll
                            for (int c4 = 0; c4 < CB / 4; ++c4) {
                                const float4 w4 = wb[(co * COS) / 4 + c4];
#pragma unroll
                                for (int i = 0; i < PM; ++i) {
                                    acc[i][4 * c4 + 0] = fmaf(a[i], w4.x, acc[i][4 * c4 + 0]);
                                    acc[i][4 * c4 + 1] = fmaf(a[i], w4.y, acc[i][4 * c4 + 1]);
                                    acc[i][4 * c4 + 2] = fmaf(a[i], w4.z, acc[i][4 * c4 + 2]);
                                    acc[i][4 * c4 + 3] = fmaf(a[i], w4.w, acc[i][4 * c4 + 3]);
                                }
                            }
                        }
                    }
                }
                const int Y = fy0 + pc + S * yq;
#pragma unroll
                for (int i = 0; i < PM; ++i) {
                    if (!okp[i]) continue;
                    const int X = fx0 + qc + S * (grp + i * Gc);
                    const bool onmap = Y >= 0 && Y < g.h && X >= 0 && X < g.w;
                    if (out_mode == OUT_CONCRETIZE) {
                        if (!onmap) continue;
                        const float* cp = centres + sp.b * (long long)g.ci * S_in + (long long)Y * g.w + X;
#pragma unroll
                        for (int c = 0; c < CB; ++c) {
                            const int ci = chunk * CB + c;
                            if (ci < g.ci) conc += fmaf(acc[i][c], cp[ci * S_in], -eps * fabsf(acc[i][c]));
                        }
                    } else {
                        const int yd = Y - doy, xd = X - dox;
                        if (yd < 0 || yd >= wd.hh || xd < 0 || xd >= wd.hw) continue;
                        float* o = out + m * ld_out + yd * wd.hw + xd;
#pragma unroll
                        for (int c = 0; c < CB; ++c) {
                            const int ci = chunk * CB + c;
                            if (ci >= g.ci) break;
                            const float v = onmap ? acc[i][c] : 0.f;
                            float* oc = o + (long long)ci * npos_d;
                            *oc = (out_mode == OUT_ACCUM) ? *oc + v : v;
                        }
                    }
                }
            }
        }
        if (active) {
            const float tot = warp_sum(cs + conc);
            if (lane == 0 && cst != nullptr) cst[m] += tot;
        }
    }
}

struct Win2Launch {
    int nwarps, HH, HW, stage_floats, w_all, ctas_per_sm, zero_fill;
    size_t smem;
    WinClasses cl;
};

template <int CB>
cudaError_t launch_back_cb(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                           const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd, int out_mode,
                           float* out, long long ld_out, float* cst, const float* centres, float eps,
                           const WinLaunch& L, cudaStream_t s) {
    const cudaError_t e = allow_dyn_smem((const void*)conv_back_win_k<CB>, kWinSmemLimit);
    if (e != cudaSuccess) return e;
    conv_back_win_k<CB><<<warp_rows_grid(M, L.nwarps, L.ctas_per_sm), 32 * L.nwarps, L.smem, s>>>(
        A, rx, ww.Wt, ww.tap_stride, ww.ci_pad, L.w_in_smem, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
        centres, eps, L.nwarps, L.stage_floats);
    return cudaGetLastError();
}

template <int S, int KS, int CB, int PM>
cudaError_t launch_back2(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                         const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd, int out_mode,
                         float* out, long long ld_out, float* cst, const float* centres, float eps,
                         const Win2Launch& L, cudaStream_t s) {
    cudaError_t e = allow_dyn_smem((const void*)conv_back_win2_k<S, KS, CB, PM>, kWinSmemLimit);
    if (e != cudaSuccess) return e;
    const float inv_hwd = 1.f / (float)wd.hw;
    int per_sm = 0;  // resident CTAs per SM (registers and shared memory)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv_back_win2_k<S, KS, CB, PM>,
                                                                  32 * L.nwarps, L.smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    conv_back_win2_k<S, KS, CB, PM><<<warp_rows_grid(M, L.nwarps, std::min(per_sm, 8)), 32 * L.nwarps, L.smem, s>>>(
        A, rx, ww.Wt, ww.tap_stride, ww.ci_pad, L.w_all, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
        centres, eps, L.nwarps, L.HH, L.HW, L.stage_floats, L.cl, inv_hwd, L.zero_fill);
    return cudaGetLastError();
}

template <int S, int KS, int CB>
cudaError_t launch_back2_pm(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                            const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd, int out_mode,
                            float* out, long long ld_out, float* cst, const float* centres, float eps,
                            const Win2Launch& L, int pm, cudaStream_t s) {
    if (pm == 4)
        return launch_back2<S, KS, CB, 4>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres,
                                          eps, L, s);
    return launch_back2<S, KS, CB, 1>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres, eps,
                                      L, s);
}

template <int S, int KS>
cudaError_t launch_back2_cb(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                            const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd, int out_mode,
                            float* out, long long ld_out, float* cst, const float* centres, float eps,
                            const Win2Launch& L, int pm, cudaStream_t s) {
    switch (ww.cb) {
        case 4:
            return launch_back2_pm<S, KS, 4>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
                                             centres, eps, L, pm, s);
        case 8:
            return launch_back2_pm<S, KS, 8>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
                                             centres, eps, L, pm, s);
        default:
            return launch_back2_pm<S, KS, 16>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst,
                                              centres, eps, L, pm, s);
    }
}

// Launch shape of the position-blocked kernel; false when (stride, taps) has no instance or a row's
// staging does not fit.
bool conv_back_win2_plan(const ConvGeom& g, const WinWeights& ww, const Win& wa, const Win& wd, int out_mode,
                         Win2Launch* L, int* pm) {
    const int S = g.stride, KS = (g.k + g.stride - 1) / g.stride;
    if (!((S == 1 && (KS == 1 || KS == 3)) || (S == 2 && (KS == 1 || KS == 2)))) return false;
    L->HH = wa.hh + KS - 1 + (g.k - 1) / S;
    L->HW = wa.hw + KS - 1 + (g.k - 1) / S;
    L->stage_floats = (wa.C * L->HH * L->HW + 3) / 4 * 4;
    const size_t stage = (size_t)L->stage_floats * sizeof(float);
    const size_t w_all = (size_t)g.k * g.k * ww.tap_stride * sizeof(float);
    const size_t w_slab = (size_t)g.k * g.k * (g.co * ww.cb + 4) * sizeof(float);
    const size_t lim = (size_t)kWinSmemLimit;
    int nw = w_all < lim ? (int)std::min<size_t>(8, (lim - w_all) / stage) : 0;
    if (nw >= 4) {
        L->w_all = 1;
        L->smem = w_all + (size_t)nw * stage;
    } else {
        if (w_slab >= lim) return false;
        nw = (int)std::min<size_t>(8, (lim - w_slab) / stage);
        if (nw < 1) return false;
        L->w_all = 0;
        L->smem = w_slab + (size_t)nw * stage;
    }
    L->nwarps = nw;
    L->ctas_per_sm = std::max(1, std::min(8, (int)(233472 / (L->smem + 1024))));
    const int NYT = S * (wa.hh - 1) + g.k, NXT = S * (wa.hw - 1) + g.k;
    *pm = (NYT * NXT >= 256) ? 4 : 1;
    int acc = 0;
    for (int pc = 0; pc < S; ++pc)
        for (int qc = 0; qc < S; ++qc) {
            const int c = pc * S + qc;
            L->cl.ny[pc] = (NYT - pc + S - 1) / S;
            L->cl.nx[qc] = (NXT - qc + S - 1) / S;
            L->cl.G[qc] = (L->cl.nx[qc] + *pm - 1) / *pm;
            L->cl.cum[c] = acc;
            acc += L->cl.ny[pc] * L->cl.G[qc];
        }
    L->cl.cum[S * S] = acc;
    for (int c = S * S + 1; c < 5; ++c) L->cl.cum[c] = acc;
    // a STORE into a destination larger than the receptive field must zero the rest of it
    const int doff_y = wd.ay == S * wa.ay ? (S * wa.by - g.pad) - wd.by : 1;
    const int doff_x = wd.ax == S * wa.ax ? (S * wa.bx - g.pad) - wd.bx : 1;
    const bool exact = doff_y == 0 && doff_x == 0 && wd.hh == NYT && wd.hw == NXT;
    L->zero_fill = (out_mode == OUT_STORE && !exact) ? 1 : 0;
    return true;
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

bool conv_back_win_whole_map_fits(const ConvGeom& g, const WinWeights& ww, const Win& wa, const Win& wd) {
    Win2Launch L;
    int pm = 1;
    return !ww.per_position && conv_back_win2_plan(g, ww, wa, wd, OUT_STORE, &L, &pm) && L.nwarps == 8 && L.w_all;
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
    Win2Launch L2;
    int pm = 1;
    if (!ww.per_position && conv_back_win2_plan(g, ww, wa, wd, out_mode, &L2, &pm)) {
        const int KS = (g.k + g.stride - 1) / g.stride;
        if (g.stride == 1 && KS == 1)
            return launch_back2_cb<1, 1>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres,
                                         eps, L2, pm, s);
        if (g.stride == 1)
            return launch_back2_cb<1, 3>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres,
                                         eps, L2, pm, s);
        if (KS == 1)
            return launch_back2_cb<2, 1>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres,
                                         eps, L2, pm, s);
        return launch_back2_cb<2, 2>(A, rx, ww, bias, M, g, pg, ps, wa, wd, out_mode, out, ld_out, cst, centres, eps,
                                     L2, pm, s);
    }
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
