// Relaxation parameters, intermediate-pass bookkeeping, specification rows, concretisation
// and the final decision: the elementwise and row-reduction kernels around the contractions.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §1 (prove the property for every input of the domain),
// §2.1 (ReLU relaxation slopes from intermediate bounds; IBP as their substitute) and §3/§4.3
// (per-neuron alpha slopes). Every row reduction here runs in a fixed order, so repeated calls
// give bitwise-identical results.
#include <mutex>
#include <set>
#include <tuple>

#include "vf_internal.cuh"

namespace vf {

namespace {

unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (unsigned)(g < 1 ? 1 : g);
}

#define GRID_STRIDE(i, n) \
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (n); i += (long long)gridDim.x * blockDim.x)

// ReLU relaxation for l <= z <= u: inactive (u <= 0, tested first) {0, 0, 0}; active (l >= 0)
// {1, 1, 0}; unstable: upper chord up = u / (u - l), t = -up * l; lower slope alpha clamped
// to [0, 1], or the adaptive choice 1 if u >= -l else 0. The fourth lane carries the bias of
// the affine node that produced z (0 if none), which the next back-substitution step adds to
// the row constant together with the relaxation intercept.
__device__ __forceinline__ float4 relax_one(float lo_b, float up_b, const float* __restrict__ alpha, long long i,
                                            float bias_v, int sound) {
    float4 p = make_float4(0.f, 0.f, 0.f, bias_v);
    if (up_b <= 0.f) {
    } else if (lo_b >= 0.f) {
        p.x = 1.f;
        p.y = 1.f;
    } else {
        const float s = up_b / (up_b - lo_b);
        p.y = s;
        // sound: the line s z + t lies above the ReLU at both ends (hence on [l, u]) in exact arithmetic
        p.z = sound ? fmaxf(__fmul_ru(s, -lo_b), __fmul_ru(up_b, __fsub_ru(1.f, s))) : -s * lo_b;
        if (alpha != nullptr)
            p.x = fminf(fmaxf(alpha[i], 0.f), 1.f);
        else
            p.x = (up_b >= -lo_b) ? 1.f : 0.f;
    }
    return p;
}

__global__ void relax_params_k(const float* __restrict__ l, const float* __restrict__ u,
                               const float* __restrict__ alpha, long long n, float4* __restrict__ P,
                               const float* __restrict__ bias, long long n_per_centre, long long per_channel,
                               int sound) {
    GRID_STRIDE(i, n) {
        const float bv = (bias != nullptr) ? bias[(i % n_per_centre) / per_channel] : 0.f;
        P[i] = relax_one(l[i], u[i], alpha, i, bv, sound);
    }
}

// One ReLU layer (n = B * n_layer neurons): its bounds and its relaxation in one pass, four neurons per
// thread (n_layer % 4 == 0). from_cr: l, u = c -/+ r as bounds_k takes them (split clamp, sound rounding)
// and stored; otherwise l, u are read and, with pass_out (the rows [I; -I] of a plain intermediate pass,
// [B, 2 n_layer]), intersected as intersect_k does on the IBP-unstable neurons and stored back. Then P as
// relax_params_k, with the same arithmetic (relax_one), so the result is bitwise the unfused one.
__global__ void relu_bounds_relax_k(const float* __restrict__ c, const float* __restrict__ r,
                                    const signed char* __restrict__ split, const float* __restrict__ pass_out,
                                    float* __restrict__ l, float* __restrict__ u, const float* __restrict__ alpha,
                                    long long n4, long long n_layer, float4* __restrict__ P,
                                    const float* __restrict__ bias, long long per_channel, int sound) {
    GRID_STRIDE(q, n4) {
        const long long i0 = 4 * q;
        float lv[4], uv[4];
        if (c != nullptr) {
            const float4 c4 = reinterpret_cast<const float4*>(c)[q], r4 = reinterpret_cast<const float4*>(r)[q];
            const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                lv[j] = sound ? __fsub_rd(cc[j], rr[j]) : cc[j] - rr[j];
                uv[j] = sound ? __fadd_ru(cc[j], rr[j]) : cc[j] + rr[j];
                if (split != nullptr) {
                    const signed char sg = split[i0 + j];
                    if (sg > 0) lv[j] = fmaxf(lv[j], 0.f);
                    if (sg < 0) uv[j] = fminf(uv[j], 0.f);
                }
            }
        } else {
            const float4 l4 = reinterpret_cast<const float4*>(l)[q], u4 = reinterpret_cast<const float4*>(u)[q];
            lv[0] = l4.x; lv[1] = l4.y; lv[2] = l4.z; lv[3] = l4.w;
            uv[0] = u4.x; uv[1] = u4.y; uv[2] = u4.z; uv[3] = u4.w;
            if (pass_out != nullptr) {
                const long long b = i0 / n_layer, j0 = i0 - b * n_layer;
                const float4 pl = *reinterpret_cast<const float4*>(pass_out + b * 2 * n_layer + j0);
                const float4 pu = *reinterpret_cast<const float4*>(pass_out + b * 2 * n_layer + n_layer + j0);
                const float ql[4] = {pl.x, pl.y, pl.z, pl.w}, qu[4] = {pu.x, pu.y, pu.z, pu.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (lv[j] < 0.f && uv[j] > 0.f) {
                        lv[j] = fmaxf(lv[j], ql[j]);
                        uv[j] = fminf(uv[j], -qu[j]);
                    }
            }
        }
        if (c != nullptr || pass_out != nullptr) {
            reinterpret_cast<float4*>(l)[q] = make_float4(lv[0], lv[1], lv[2], lv[3]);
            reinterpret_cast<float4*>(u)[q] = make_float4(uv[0], uv[1], uv[2], uv[3]);
        }
        const long long j0 = i0 % n_layer;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float bv = (bias != nullptr) ? bias[(j0 + j) / per_channel] : 0.f;
            P[i0 + j] = relax_one(lv[j], uv[j], alpha, i0 + j, bv, sound);
        }
    }
}

// Identity-trick start of an intermediate pass over node p (n_p neurons, rows [I; -I]):
// the first back-substitution step through p adds +-b_p[j] to row j's constant.
__global__ void cst_identity_bias_k(float* __restrict__ cst, long long M, PassGeom pg, const float* __restrict__ bias,
                                    long long n_p, long long per_channel) {
    GRID_STRIDE(m, M) {
        float sg;
        const long long j = start_neuron(pg, n_p, m, &sg);
        cst[m] += sg * bias[j / per_channel];
    }
}

__global__ void ident_rows_k(float* __restrict__ out, long long ld, long long M, PassGeom pg, long long n_p,
                             int accumulate) {
    GRID_STRIDE(e, M * n_p) {
        const long long m = e / n_p, c = e % n_p;
        float sg;
        const long long j = start_neuron(pg, n_p, m, &sg);
        const float v = (c == j) ? sg : 0.f;
        float* o = out + m * ld + c;
        *o = accumulate ? (*o + v) : v;
    }
}

// Rows +-(row j of the convolution's matrix) over the conv's input: the identity-trick first
// step of an intermediate pass that starts at a convolution. One CTA per row.
__global__ void conv_start_rows_k(float* __restrict__ out, long long ld, long long M, PassGeom pg,
                                  const float* __restrict__ W, ConvGeom g, int accumulate) {
    const long long n_p = (long long)g.co * g.ho * g.wo;
    const long long nin = (long long)g.ci * g.h * g.w;
    for (long long m = blockIdx.x; m < M; m += gridDim.x) {
        float* o = out + m * ld;
        if (!accumulate) {
            for (long long c = threadIdx.x; c < nin; c += blockDim.x) o[c] = 0.f;
            __syncthreads();
        }
        float sg;
        const long long j = start_neuron(pg, n_p, m, &sg);
        const int co = (int)(j / (g.ho * g.wo));
        const int oi = (int)((j / g.wo) % g.ho);
        const int oj = (int)(j % g.wo);
        const int nk = g.ci * g.k * g.k;
        for (int e = threadIdx.x; e < nk; e += blockDim.x) {
            const int q = e % g.k, p = (e / g.k) % g.k, ci = e / (g.k * g.k);
            const int y = oi * g.stride - g.pad + p, x = oj * g.stride - g.pad + q;
            if (y < 0 || y >= g.h || x < 0 || x >= g.w) continue;
            o[((long long)ci * g.h + y) * g.w + x] += sg * W[(((long long)co * g.ci + ci) * g.k + p) * g.k + q];
        }
        __syncthreads();
    }
}

__device__ __forceinline__ float block_sum256(float v, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0)
        for (int i = 0; i < 8; ++i) t += red[i];
    __syncthreads();
    return t;
}

// out[m, :] (=, +=) relax(A[m, :]); cst[m] += relaxation constant. One CTA per row; may run
// in place (each element is read and written by the same thread).
__global__ void __launch_bounds__(256)
relax_rows_k(RowRef A, Relax rx, long long M, int n, PassGeom pg, float* out, long long ld_out, int accumulate,
             float* __restrict__ cst) {
    __shared__ float red[8];
    for (long long m = blockIdx.x; m < M; m += gridDim.x) {
        const float* a = A.row(m);
        const long long b = (pg.pass_m0 + m) / pg.R_pass;
        float* o = out + m * ld_out;
        float cs = 0.f;
        for (int j = threadIdx.x; j < n; j += 256) {
            const float x = a[j];
            float r = x;
            if (rx.P != nullptr) {
                const float4 p = rx.P[b * n + j];
                r = (x >= 0.f) ? x * p.x : x * p.y;
                if (rx.count_const) cs = fmaf(fminf(x, 0.f), p.z, cs);
            }
            o[j] = accumulate ? (o[j] + r) : r;
        }
        if (rx.P != nullptr && rx.count_const && cst != nullptr) {
            const float t = block_sum256(cs, red);
            if (threadIdx.x == 0) cst[m] += t;
        }
    }
}

// cst[m] += A[m, :] . c_b - eps * |A[m, :]|_1 : concretisation of materialised input rows.
__global__ void __launch_bounds__(256)
concretize_rows_k(RowRef A, long long M, int n0, PassGeom pg, const float* __restrict__ centres, float eps,
                  float* __restrict__ cst) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * 8;
    for (long long m = blockIdx.x * 8LL + (threadIdx.x >> 5); m < M; m += warps) {
        const float* a = A.row(m);
        const float* c = centres + ((pg.pass_m0 + m) / pg.R_pass) * (long long)n0;
        float s = 0.f;
        for (int i = lane; i < n0; i += 32) s += fmaf(a[i], c[i], -eps * fabsf(a[i]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) cst[m] += s;
    }
}

__global__ void finish_rows_k(const float* __restrict__ cst, const float* __restrict__ part, int ntiles, long long M,
                              float* __restrict__ out) {
    GRID_STRIDE(m, M) {
        float v = cst[m];
        for (int t = 0; t < ntiles; ++t) v += part[(long long)t * M + m];
        out[m] = v;
    }
}

__global__ void add_partials_k(float* __restrict__ cst, const float* __restrict__ part, int ntiles, long long M) {
    GRID_STRIDE(m, M) {
        float v = 0.f;
        for (int t = 0; t < ntiles; ++t) v += part[(long long)t * M + m];
        cst[m] += v;
    }
}

// Intermediate bounds after a pass over node p (rows [I; -I] per centre): IBP-unstable neurons
// take l = max(l, lb_j), u = min(u, -lb_{n + j}); IBP-stable ones keep their (exact) relaxation.
__global__ void intersect_k(float* __restrict__ l, float* __restrict__ u, const float* __restrict__ pass_out, int B,
                            long long n) {
    GRID_STRIDE(i, (long long)B * n) {
        const long long b = i / n, j = i % n;
        const float l0 = l[i], u0 = u[i];
        if (l0 < 0.f && u0 > 0.f) {
            l[i] = fmaxf(l0, pass_out[b * 2 * n + j]);
            u[i] = fminf(u0, -pass_out[b * 2 * n + n + j]);
        }
    }
}

// Unstable-neuron compaction (rows of an intermediate pass only for IBP-unstable neurons: the others keep
// their IBP bounds, so their rows are never used). One CTA of 256 threads per centre.
__global__ void __launch_bounds__(256) unstable_count_k(const float* __restrict__ l, const float* __restrict__ u,
                                                        long long n, int* __restrict__ counts) {
    __shared__ int red[8];
    const long long b = blockIdx.x;
    int c = 0;
    for (long long j = threadIdx.x; j < n; j += 256) c += (l[b * n + j] < 0.f && u[b * n + j] > 0.f) ? 1 : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int i = 0; i < 8; ++i) t += red[i];
        counts[b] = t;
    }
}

// idx[b * half + i] = the i-th unstable neuron of centre b (increasing order), -1 for i >= its count.
// Each 256-neuron chunk is ranked with warp ballots and a prefix over the 8 warps.
__global__ void __launch_bounds__(256) unstable_list_k(const float* __restrict__ l, const float* __restrict__ u,
                                                       long long n, int half, int* __restrict__ idx) {
    __shared__ int wcount[8];
    __shared__ int base_sh;
    const long long b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) base_sh = 0;
    __syncthreads();
    for (long long j0 = 0; j0 < n; j0 += 256) {
        const long long j = j0 + threadIdx.x;
        const bool un = j < n && l[b * n + j] < 0.f && u[b * n + j] > 0.f;
        const unsigned bal = __ballot_sync(0xffffffffu, un);
        if (lane == 0) wcount[warp] = __popc(bal);
        __syncthreads();
        int before = base_sh;
        for (int w = 0; w < warp; ++w) before += wcount[w];
        const int pos = before + __popc(bal & ((1u << lane) - 1u));
        if (un && pos < half) idx[b * half + pos] = (int)j;
        __syncthreads();
        if (threadIdx.x == 0) {
            int t = 0;
            for (int w = 0; w < 8; ++w) t += wcount[w];
            base_sh += t;
        }
        __syncthreads();
    }
    for (int i = base_sh + threadIdx.x; i < half; i += 256) idx[b * half + i] = -1;
}

// Intersection after a compacted pass (2 * half rows per centre: +e_j for the listed j, then -e_j).
__global__ void intersect_compact_k(float* __restrict__ l, float* __restrict__ u, const float* __restrict__ pass_out,
                                    const int* __restrict__ idx, int B, long long n, int half) {
    GRID_STRIDE(e, (long long)B * half) {
        const long long b = e / half, i = e % half;
        const int j = idx[e];
        if (j < 0) continue;
        const long long k = b * n + j;
        l[k] = fmaxf(l[k], pass_out[b * 2 * half + i]);
        u[k] = fminf(u[k], -pass_out[b * 2 * half + half + i]);
    }
}

// out[m, :] = sg * W[j, :] for the start neuron j of row m (compacted pass over a dense node).
__global__ void gather_start_rows_k(float* __restrict__ out, long long ld, long long M, PassGeom pg,
                                    const float* __restrict__ W, long long n_p, long long n_src) {
    for (long long m = blockIdx.x; m < M; m += gridDim.x) {
        float sg;
        const long long j = start_neuron(pg, n_p, m, &sg);
        const float* w = W + j * n_src;
        float* o = out + m * ld;
        for (long long c = threadIdx.x; c < n_src; c += blockDim.x) o[c] = sg * w[c];
    }
}

__global__ void spec_rows_k(const float* __restrict__ C, long long C_bstride, int BC, int R, int nL,
                            float* __restrict__ S) {
    GRID_STRIDE(e, (long long)BC * R * nL) {
        const long long bc = e / ((long long)R * nL);
        const long long rest = e % ((long long)R * nL);
        const float v = C[bc * C_bstride + rest];
        S[bc * 2LL * R * nL + rest] = v;
        S[bc * 2LL * R * nL + (long long)R * nL + rest] = -v;
    }
}

// IBP bound of the specification: C applied to the last node's interval, C c -+ |C| r.
__global__ void __launch_bounds__(256)
spec_ibp_k(const float* __restrict__ C, long long C_bstride, int B, int R, int nL, const float* __restrict__ zc,
           const float* __restrict__ zr, float* __restrict__ lb, float* __restrict__ ub, float gam) {
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * R;
    for (long long w = blockIdx.x * 8LL + (threadIdx.x >> 5); w < rows; w += (long long)gridDim.x * 8) {
        const long long b = w / R, r = w % R;
        const float* cr = C + b * C_bstride + r * nL;
        float sc = 0.f, sr = 0.f, sa = 0.f;
        for (int j = lane; j < nL; j += 32) {
            sc = fmaf(cr[j], zc[b * nL + j], sc);
            sr = fmaf(fabsf(cr[j]), zr[b * nL + j], sr);
            if (gam > 0.f) sa = __fmaf_ru(fabsf(cr[j]), __fadd_ru(fabsf(zc[b * nL + j]), zr[b * nL + j]), sa);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sc += __shfl_xor_sync(0xffffffffu, sc, off);
            sr += __shfl_xor_sync(0xffffffffu, sr, off);
            sa = __fadd_ru(sa, __shfl_xor_sync(0xffffffffu, sa, off));
        }
        if (lane == 0) {
            if (gam > 0.f) {  // sound: both sums err by at most gam * sum |C| (|zc| + zr)
                const float e = __fmul_ru(gam, sa);
                lb[w] = __fsub_rd(__fsub_rd(sc, sr), e);
                ub[w] = __fadd_ru(__fadd_ru(sc, sr), e);
            } else {
                lb[w] = sc - sr;
                ub[w] = sc + sr;
            }
        }
    }
}

__global__ void decide_k(const float* __restrict__ lb_ibp, const float* __restrict__ ub_ibp,
                         const float* __restrict__ pass_out, int B, int R, int both, float* __restrict__ lb,
                         float* __restrict__ ub, float* __restrict__ lb_ibp_out, uint8_t* __restrict__ verified) {
    GRID_STRIDE(i, (long long)B * R) {
        const long long b = i / R, r = i % R;
        const long long Rp = both ? 2LL * R : (long long)R;
        const float l = fmaxf(lb_ibp[i], pass_out[b * Rp + r]);
        lb[i] = l;
        if (both) ub[i] = fminf(ub_ibp[i], -pass_out[b * Rp + R + r]);
        if (lb_ibp_out != nullptr) lb_ibp_out[i] = lb_ibp[i];
        if (verified != nullptr) verified[i] = (l > 0.f) ? 1 : 0;
    }
}

__global__ void finite_scan_k(const float* __restrict__ p, long long n, int* flag) {
    GRID_STRIDE(i, n) {
        if (!isfinite(p[i])) atomicOr(flag, 1);
    }
}

__global__ void __launch_bounds__(256)
concretize_api_k(const float* __restrict__ lambda, const float* __restrict__ cst, const float* __restrict__ centres,
                 float eps, int B, int R, int n0, float* __restrict__ lb) {
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * R;
    for (long long w = blockIdx.x * 8LL + (threadIdx.x >> 5); w < rows; w += (long long)gridDim.x * 8) {
        const float* a = lambda + w * n0;
        const float* c = centres + (w / R) * (long long)n0;
        float s = 0.f;
        for (int i = lane; i < n0; i += 32) s += fmaf(a[i], c[i], -eps * fabsf(a[i]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) lb[w] = s + (cst != nullptr ? cst[w] : 0.f);
    }
}

unsigned rows_grid(long long rows_per_cta_units) {
    long long g = rows_per_cta_units;
    if (g > 148LL * 16) g = 148LL * 16;
    return (unsigned)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_relax_params(const float* l, const float* u, const float* alpha, long long n, float4* P,
                                const float* bias, long long n_per_centre, long long per_channel, cudaStream_t s,
                                int sound) {
    relax_params_k<<<grid_for(n, 256), 256, 0, s>>>(l, u, alpha, n, P, bias, n_per_centre, per_channel, sound);
    return cudaGetLastError();
}

cudaError_t launch_relu_bounds_relax(const float* c, const float* r, const signed char* split, const float* pass_out,
                                     float* l, float* u, const float* alpha, int B, long long n_layer, float4* P,
                                     const float* bias, long long per_channel, int sound, cudaStream_t s) {
    const long long n = (long long)B * n_layer;
    if (n_layer % 4 != 0 || (reinterpret_cast<uintptr_t>(l) & 15) || (reinterpret_cast<uintptr_t>(u) & 15) ||
        (c && ((reinterpret_cast<uintptr_t>(c) & 15) || (reinterpret_cast<uintptr_t>(r) & 15))) ||
        (pass_out && (reinterpret_cast<uintptr_t>(pass_out) & 15))) {
        // unvectorisable layout: the two unfused steps
        cudaError_t e = cudaSuccess;
        if (c != nullptr) e = launch_bounds_from_cr(c, r, n, l, u, s, split, sound);
        else if (pass_out != nullptr) e = launch_intersect(l, u, nullptr, nullptr, pass_out, B, n_layer, s);
        if (e != cudaSuccess) return e;
        return launch_relax_params(l, u, alpha, n, P, bias, n_layer, per_channel, s, sound);
    }
    relu_bounds_relax_k<<<grid_for(n / 4, 256), 256, 0, s>>>(c, r, split, pass_out, l, u, alpha, n / 4, n_layer, P,
                                                            bias, per_channel, sound);
    return cudaGetLastError();
}

cudaError_t launch_cst_identity_bias(float* cst, long long M, PassGeom pg, const float* bias, long long n_p,
                                     long long per_channel, cudaStream_t s) {
    cst_identity_bias_k<<<grid_for(M, 256), 256, 0, s>>>(cst, M, pg, bias, n_p, per_channel);
    return cudaGetLastError();
}

cudaError_t launch_ident_rows(float* out, long long ld, long long M, PassGeom pg, long long n_p, int accumulate,
                              cudaStream_t s) {
    ident_rows_k<<<grid_for(M * n_p, 256), 256, 0, s>>>(out, ld, M, pg, n_p, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_conv_start_rows(float* out, long long ld, long long M, PassGeom pg, const float* W,
                                   const ConvGeom& g, int accumulate, cudaStream_t s) {
    conv_start_rows_k<<<rows_grid(M), 256, 0, s>>>(out, ld, M, pg, W, g, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_relax_rows(const RowRef& A, Relax rx, long long M, int n, PassGeom pg, float* out,
                              long long ld_out, int accumulate, float* cst, cudaStream_t s) {
    relax_rows_k<<<rows_grid(M), 256, 0, s>>>(A, rx, M, n, pg, out, ld_out, accumulate, cst);
    return cudaGetLastError();
}

cudaError_t launch_concretize_rows(const RowRef& A, long long M, int n0, PassGeom pg, const float* centres, float eps,
                                   float* cst, cudaStream_t s) {
    concretize_rows_k<<<rows_grid((M + 7) / 8), 256, 0, s>>>(A, M, n0, pg, centres, eps, cst);
    return cudaGetLastError();
}

cudaError_t launch_finish_rows(const float* cst, const float* part, int ntiles, long long M, float* out,
                               cudaStream_t s) {
    finish_rows_k<<<grid_for(M, 256), 256, 0, s>>>(cst, part, ntiles, M, out);
    return cudaGetLastError();
}

cudaError_t launch_add_partials(float* cst, const float* part, int ntiles, long long M, cudaStream_t s) {
    add_partials_k<<<grid_for(M, 256), 256, 0, s>>>(cst, part, ntiles, M);
    return cudaGetLastError();
}

cudaError_t launch_intersect(float* l, float* u, const float* l_ibp, const float* u_ibp, const float* pass_out, int B,
                             long long n, cudaStream_t s) {
    (void)l_ibp;
    (void)u_ibp;
    intersect_k<<<grid_for((long long)B * n, 256), 256, 0, s>>>(l, u, pass_out, B, n);
    return cudaGetLastError();
}

cudaError_t launch_unstable_count(const float* l, const float* u, int B, long long n, int* counts, cudaStream_t s) {
    if (B <= 0) return cudaSuccess;
    unstable_count_k<<<B, 256, 0, s>>>(l, u, n, counts);
    return cudaGetLastError();
}

cudaError_t launch_unstable_list(const float* l, const float* u, int B, long long n, int half, int* idx, cudaStream_t s) {
    if (B <= 0 || half <= 0) return cudaSuccess;
    unstable_list_k<<<B, 256, 0, s>>>(l, u, n, half, idx);
    return cudaGetLastError();
}

cudaError_t launch_intersect_compact(float* l, float* u, const float* pass_out, const int* idx, int B, long long n,
                                     int half, cudaStream_t s) {
    if (B <= 0 || half <= 0) return cudaSuccess;
    intersect_compact_k<<<grid_for((long long)B * half, 256), 256, 0, s>>>(l, u, pass_out, idx, B, n, half);
    return cudaGetLastError();
}

cudaError_t launch_gather_start_rows(float* out, long long ld, long long M, PassGeom pg, const float* W, long long n_p,
                                     long long n_src, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    gather_start_rows_k<<<rows_grid(M), 256, 0, s>>>(out, ld, M, pg, W, n_p, n_src);
    return cudaGetLastError();
}

cudaError_t launch_spec_rows(const float* C, long long C_bstride, int BC, int R, int nL, float* S, cudaStream_t s) {
    spec_rows_k<<<grid_for((long long)BC * R * nL, 256), 256, 0, s>>>(C, C_bstride, BC, R, nL, S);
    return cudaGetLastError();
}

cudaError_t launch_spec_ibp(const float* C, long long C_bstride, int B, int R, int nL, const float* zc, const float* zr,
                            float* lb, float* ub, cudaStream_t s, float gam) {
    spec_ibp_k<<<rows_grid(((long long)B * R + 7) / 8), 256, 0, s>>>(C, C_bstride, B, R, nL, zc, zr, lb, ub, gam);
    return cudaGetLastError();
}

cudaError_t launch_decide(const float* lb_ibp, const float* ub_ibp, const float* pass_out, int B, int R, int both,
                          float* lb, float* ub, float* lb_ibp_out, uint8_t* verified, cudaStream_t s) {
    decide_k<<<grid_for((long long)B * R, 256), 256, 0, s>>>(lb_ibp, ub_ibp, pass_out, B, R, both, lb, ub, lb_ibp_out,
                                                             verified);
    return cudaGetLastError();
}

cudaError_t launch_finite_scan(const float* p, long long n, int* flag, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    finite_scan_k<<<grid_for(n, 256), 256, 0, s>>>(p, n, flag);
    return cudaGetLastError();
}

cudaError_t launch_concretize_api(const float* lambda, const float* cst, const float* centres, float eps, int B, int R,
                                  int n0, float* lb, cudaStream_t s) {
    concretize_api_k<<<rows_grid(((long long)B * R + 7) / 8), 256, 0, s>>>(lambda, cst, centres, eps, B, R, n0, lb);
    return cudaGetLastError();
}

cudaError_t allow_dyn_smem(const void* func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::set<std::tuple<const void*, int, int>> done;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(func, dev, bytes);
    if (done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert(key);
    return e;
}

}  // namespace vf
