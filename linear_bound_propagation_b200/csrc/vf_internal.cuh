// Internal declarations shared by the CUDA kernels (k_*.cu) and the host executor (vf_api.cu).
// Nothing here is part of the public ABI (include/vf.h).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace vf {

// Read-only addressing of coefficient rows. Local row m of a launch maps to global
// row g = m + m0, stored at ptr + (g / RA) * sB + (g % RA) * ld. A chunk-local buffer
// uses m0 = 0, sB = 0, RA = kHugeRows; a block shared by all centres (the [W; -W] start
// rows of an intermediate pass, or a specification matrix C with centre stride 0) uses
// m0 = the chunk's first global row, RA = rows per centre and sB = 0 (or the C stride).
constexpr long long kHugeRows = (1LL << 62);

struct RowRef {
    const float* ptr;
    long long sB, ld, RA, m0;
    __host__ __device__ __forceinline__ const float* row(long long m) const {
        long long g = m + m0;
        return ptr + (g / RA) * sB + (g % RA) * ld;
    }
};

// ReLU relaxation applied to coefficients as they are loaded: P[b * n + j] holds
// {lo, up, t, 0} for centre b and neuron j (lower slope used by coefficients >= 0,
// upper slope and intercept used by coefficients < 0). P == nullptr: no relaxation.
struct Relax {
    const float4* P;
    int count_const;  // also add sum_j min(x_j, 0) * t_j to the row constant
};

// Rows of one CROWN pass are processed in chunks; row m of a chunk is global row
// pass_m0 + m, which belongs to centre (pass_m0 + m) / R_pass.
struct PassGeom {
    long long pass_m0;
    long long R_pass;
    const int* idx = nullptr;  // compacted identity-trick pass: start neurons, see start_neuron
};

// Start neuron of local row m of an identity-trick pass over a node with n_start neurons. Plain pass:
// rows [I; -I] per centre. Compacted pass (pg.idx set): rows [e_j; -e_j] for the neurons listed in
// idx[b * (R_pass / 2) + i]; a padding slot holds -1 and stands for neuron 0 (its result is unused).
__device__ __forceinline__ long long start_neuron(const PassGeom& pg, long long n_start, long long m, float* sg) {
    const long long g = pg.pass_m0 + m;
    const long long r = g % pg.R_pass;
    if (pg.idx == nullptr) {
        *sg = (r < n_start) ? 1.f : -1.f;
        return r % n_start;
    }
    const long long half = pg.R_pass >> 1;
    *sg = (r < half) ? 1.f : -1.f;
    const int j = pg.idx[(g / pg.R_pass) * half + (r % half)];
    return j < 0 ? 0 : j;
}

enum OutMode { OUT_STORE = 0, OUT_ACCUM = 1, OUT_CONCRETIZE = 2 };

struct ConvGeom {
    int ci, h, w;     // input (source) shape
    int co, ho, wo;   // output shape
    int k, stride, pad;
};

// ---- contractions (k_back.cu, k_back_conv.cu) ----------------------------------------
// out[m, :] (=, +=) relax(A[m, :]) . W  with W = the node's [K = n_out, N = n_in] weights;
// cst[m] += sum_k (relax const) + relax(A)[m, k] * bias[k]   (when cst != nullptr);
// OUT_CONCRETIZE: part[tile_n * M + m] = sum_{n in tile} v * c_b[n] - eps * |v|.
int dense_back_tiles_n(int N);
cudaError_t launch_dense_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M, int K,
                              int N, PassGeom pg, int out_mode, float* out, long long ld_out, float* cst,
                              const float* centres, float eps, float* part, cudaStream_t s);

// Transposed convolution of relaxed rows over the conv output back onto its input. Writes per-tile
// partials cpart[tile * M + m] (tile < conv_back_tiles(g)) holding the row-constant terms the tile owns
// and, with OUT_CONCRETIZE, the tile's concretised outputs; launch_add_partials folds them into cst.
size_t conv_back_smem_bytes(const ConvGeom& g);
int conv_back_tiles(const ConvGeom& g);
bool conv_back_supported(const ConvGeom& g);
cudaError_t launch_conv_back(const RowRef& A, Relax rx, const float* W, const float* bias, long long M,
                             const ConvGeom& g, PassGeom pg, int out_mode, float* out, long long ld_out, float* cpart,
                             const float* centres, float eps, int num_sms, cudaStream_t s);

// ---- receptive-field windows (k_win.cu) ----------------------------------------------
// In a pass that starts at a convolution node p, the row of start neuron j = (c_j, y_j, x_j) is nonzero
// only inside the receptive field of (y_j, x_j) on every map below p. Such rows are stored as a window
// [C][hh][hw] whose origin on the map is (ay * y_j + by, ax * x_j + bx). Entries that fall outside the
// map are held as zeros. ay = ax = by = bx = 0 with hh, hw the map's height and width is the whole map,
// i.e. the plain row layout.
struct Win {
    int C, hh, hw;
    int ay, by, ax, bx;
};
// The start node of the pass: neurons per centre, output height and width. Row r of a centre starts
// from +e_j (r < n) or -e_j (r >= n), j = r mod n.
struct PassStart {
    long long n;
    int h, w;
};
// Start rows +-(row j of the convolution's matrix) over the convolution's input, written into window
// `wd`, which must contain the k x k field of every start neuron.
cudaError_t launch_conv_start_rows_win(float* out, long long ld, long long M, PassGeom pg, PassStart ps, const float* W,
                                       const ConvGeom& g, const Win& wd, int accumulate, cudaStream_t s);
// Weights of a convolution in the layout of the windowed transposed convolution: tap (p, q) at
// Wt + (p * k + q) * tap_stride holds [co][ci_pad] (ci padded to a multiple of cb, the input channels a
// thread accumulates at once); tap_stride = co * ci_pad + 4 floats.
struct WinWeights {
    const float* Wt;
    int tap_stride, ci_pad, cb;
    int per_position;  // 1: always the per-position kernel (no position blocking)
};
int win_ci_block(int ci);
constexpr int kWinSmemLimit = 220 * 1024;
struct WinLaunch {
    int nwarps, stage_floats, w_in_smem, ctas_per_sm;
    size_t smem;
};
// Launch shape of the windowed transposed convolution for rows in window `wa`; false when one row's
// staging does not fit in shared memory.
bool conv_back_win_plan(const ConvGeom& g, const WinWeights& ww, const Win& wa, WinLaunch* L);
// Transposed convolution of windowed rows: A over the conv output in window `wa` (relaxed on load by rx,
// bias added to cst) onto the conv input in window `wd` (which must contain the receptive field of `wa`).
// OUT_CONCRETIZE adds the concretised rows to cst instead of storing them. cst[m] receives one sum per
// launch and row.
cudaError_t launch_conv_back_win(const RowRef& A, Relax rx, const WinWeights& ww, const float* bias, long long M,
                                 const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                 int out_mode, float* out, long long ld_out, float* cst, const float* centres, float eps,
                                 cudaStream_t s);
// Identity start rows +-e_j written into window `wd` (which must contain position (y_j, x_j)) of a map with
// the start node's shape.
cudaError_t launch_ident_rows_win(float* out, long long ld, long long M, PassGeom pg, PassStart ps, const Win& wd,
                                  int accumulate, cudaStream_t s);
// True when rows over the whole map (`wa` = the whole output map, `wd` = the whole input map) fit the
// position-blocked windowed kernel with a full CTA of 8 rows and all weights in shared memory; such
// convolutions run faster there than in the tiled whole-map kernel.
bool conv_back_win_whole_map_fits(const ConvGeom& g, const WinWeights& ww, const Win& wa, const Win& wd);
// Re-windowing of rows over one map of C x H x W: out (=, +=) relax(A) moved from window `wa` into `wd`
// (which must contain `wa`); relaxation constants (rx.count_const) go to cst.
cudaError_t launch_rewin_rows(const RowRef& A, Relax rx, long long M, int C, int H, int W, PassGeom pg, PassStart ps,
                              const Win& wa, const Win& wd, float* out, long long ld_out, int accumulate, float* cst,
                              cudaStream_t s);

// ---- tensor-core convolution (k_back_conv_tc.cu) ----------------------------------------
// The same step as launch_conv_back_win (rows over the conv output in window wa, relaxed on load, bias into
// cst; out in window wd, or concretised into cst), as a tcgen05 implicit GEMM (3xTF32). Whole-map rows are
// the window of the whole map (ay = ax = by = bx = 0). Conditions: C_in a multiple of 16 up to 128, k <= 8,
// stride 1 or 2, and one row's shifted slabs within the TMEM and shared-memory plan. A STORE writes every entry
// of wd only when conv_back_tc_covers(g, wa, wd); otherwise the caller clears the rows first. Writes *err on
// a bounded-wait expiry.
bool conv_tc_weights_supported(const ConvGeom& g);
int conv_tc_wtc_floats(const ConvGeom& g);
void conv_tc_pack_weights(const ConvGeom& g, const float* W, float* out);
bool conv_back_tc_supported(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode);
bool conv_back_tc_covers(const ConvGeom& g, const Win& wa, const Win& wd);
cudaError_t launch_conv_back_tc(const RowRef& A, Relax rx, const float* Wtc, const float* bias, long long M,
                                const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                int out_mode, float* out, long long ld_out, float* cst, const float* centres,
                                float eps, int* err, int num_sms, cudaStream_t s);

// ---- tensor-core convolution with the taps in N (k_back_conv_tcn.cu) ------------------------
// The same step as launch_conv_back_tc with one GEMM column per (tap, input channel): three large MMAs per tile
// and 8 output channels; the taps are summed in shared memory. Conditions: C_in a multiple of 16, C_in k^2 <= 512
// in at most four groups of <= 256 columns, k <= 8, and one row's natural window within shared memory.
// conv_tcn_wtn_floats is 0 when the weights do not fit the scheme. The same coverage rule as
// conv_back_tc_covers applies to STOREs.
int conv_tcn_wtn_floats(const ConvGeom& g);
void conv_tcn_pack_weights(const ConvGeom& g, const float* W, float* out);
bool conv_back_tcn_supported(const ConvGeom& g, const Win& wa, const Win& wd, int out_mode);
cudaError_t launch_conv_back_tcn(const RowRef& A, Relax rx, const float* Wtn, const float* bias, long long M,
                                 const ConvGeom& g, PassGeom pg, PassStart ps, const Win& wa, const Win& wd,
                                 int out_mode, float* out, long long ld_out, float* cst, const float* centres,
                                 float eps, int* err, int num_sms, cudaStream_t s);

// ---- IBP (k_ibp.cu) -------------------------------------------------------------------
// rowsum_abs (optional): sum_k |W[n, k]|, used with `eps` when the source is the input box (radius eps everywhere).
cudaError_t launch_ibp_dense(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                             const float* rowsum_abs, float eps, int B, int K, int N, float* zc, float* zr,
                             cudaStream_t s);
// hr and zr may both be NULL: then only the centre map W * hc + b is computed (the alpha-CROWN gradient).
// zr[m, n] = eps * rowsum_abs[n] for m < B: the IBP radius of a dense layer fed by the input box.
cudaError_t launch_ibp_radius_rowsum(const float* rowsum_abs, float eps, int B, int N, float* zr, cudaStream_t s);
cudaError_t launch_ibp_conv(const float* hc, const float* hr, const float* W, const float* Wabs, const float* bias,
                            int B, const ConvGeom& g, float* zc, float* zr, cudaStream_t s);
cudaError_t launch_ibp_relu(const float* c, const float* r, long long n, float* oc, float* orad, cudaStream_t s,
                            const signed char* split = nullptr);
cudaError_t launch_ibp_add(const float* c1, const float* r1, const float* c2, const float* r2, long long n,
                           float* oc, float* orad, cudaStream_t s);
cudaError_t launch_fill(float* p, long long n, float v, cudaStream_t s);
cudaError_t launch_bounds_from_cr(const float* c, const float* r, long long n, float* lb, float* ub, cudaStream_t s,
                                  const signed char* split = nullptr, int sound = 0);
// out = A |W|^T (A [M, K], Wabs [N, K] = |W|): the radius half of the dense interval product.
cudaError_t launch_abs_rows_times_wt(const float* A, const float* Wabs, int M, int K, int N, float* out, cudaStream_t s);

// ---- relaxation, pass bookkeeping, decision (k_misc.cu) ------------------------------
// P[i] = {lo, up, t, bias of the affine source}; bias may be null (then 0); neuron j = i % n_per_centre
// takes bias[j / per_channel] (per_channel = H*W for a convolution, 1 for a dense node).
// sound != 0: the intercept t is rounded up so that the upper line stays above the ReLU at both ends.
cudaError_t launch_relax_params(const float* l, const float* u, const float* alpha, long long n, float4* P,
                                const float* bias, long long n_per_centre, long long per_channel, cudaStream_t s,
                                int sound = 0);
// One ReLU layer's bounds and relaxation in one pass over its B * n_layer neurons: bounds from the IBP
// centre/radius (c, r given; as launch_bounds_from_cr) or read from l, u and intersected with a plain
// pass's rows (pass_out given; as launch_intersect), then P as launch_relax_params. Falls back to those
// launches when n_layer is not a multiple of 4 or an array is not 16-byte aligned.
cudaError_t launch_relu_bounds_relax(const float* c, const float* r, const signed char* split, const float* pass_out,
                                     float* l, float* u, const float* alpha, int B, long long n_layer, float4* P,
                                     const float* bias, long long per_channel, int sound, cudaStream_t s);
cudaError_t launch_cst_identity_bias(float* cst, long long M, PassGeom pg, const float* bias, long long n_p,
                                     long long per_channel, cudaStream_t s);
cudaError_t launch_ident_rows(float* out, long long ld, long long M, PassGeom pg, long long n_p, int accumulate,
                              cudaStream_t s);
cudaError_t launch_conv_start_rows(float* out, long long ld, long long M, PassGeom pg, const float* W,
                                   const ConvGeom& g, int accumulate, cudaStream_t s);
cudaError_t launch_relax_rows(const RowRef& A, Relax rx, long long M, int n, PassGeom pg, float* out, long long ld_out,
                              int accumulate, float* cst, cudaStream_t s);
cudaError_t launch_concretize_rows(const RowRef& A, long long M, int n0, PassGeom pg, const float* centres, float eps,
                                   float* cst, cudaStream_t s);
cudaError_t launch_finish_rows(const float* cst, const float* part, int ntiles, long long M, float* out,
                               cudaStream_t s);
// cst[m] += sum_{t < ntiles} part[t * M + m], in increasing t.
cudaError_t launch_add_partials(float* cst, const float* part, int ntiles, long long M, cudaStream_t s);
cudaError_t launch_intersect(float* l, float* u, const float* l_ibp, const float* u_ibp, const float* pass_out,
                             int B, long long n, cudaStream_t s);
// Unstable-neuron compaction of an intermediate pass (IBP bounds l < 0 < u): counts[b] = number of such
// neurons of centre b; idx[b * half + i] = the i-th of them in increasing order, -1 past the count.
cudaError_t launch_unstable_count(const float* l, const float* u, int B, long long n, int* counts, cudaStream_t s);
cudaError_t launch_unstable_list(const float* l, const float* u, int B, long long n, int half, int* idx, cudaStream_t s);
// Intersection for a compacted pass: rows [e_j; -e_j] of the listed neurons, R = 2 * half rows per centre.
cudaError_t launch_intersect_compact(float* l, float* u, const float* pass_out, const int* idx, int B, long long n,
                                     int half, cudaStream_t s);
// Rows +-W[j, :] (W is [n_p, n_src], row-major) for the start neurons of a compacted pass over a dense node.
cudaError_t launch_gather_start_rows(float* out, long long ld, long long M, PassGeom pg, const float* W, long long n_p,
                                     long long n_src, cudaStream_t s);
cudaError_t launch_spec_rows(const float* C, long long C_bstride, int BC, int R, int nL, float* S, cudaStream_t s);
// gam > 0: sound mode, both bounds widened by gam * sum |C| (|zc| + zr) and rounded outwards.
cudaError_t launch_spec_ibp(const float* C, long long C_bstride, int B, int R, int nL, const float* zc, const float* zr,
                            float* lb, float* ub, cudaStream_t s, float gam = 0.f);
cudaError_t launch_decide(const float* lb_ibp, const float* ub_ibp, const float* pass_out, int B, int R, int both,
                          float* lb, float* ub, float* lb_ibp_out, uint8_t* verified, cudaStream_t s);
cudaError_t launch_finite_scan(const float* p, long long n, int* flag, cudaStream_t s);
cudaError_t launch_concretize_api(const float* lambda, const float* cst, const float* centres, float eps, int B, int R,
                                  int n0, float* lb, cudaStream_t s);

// out[m, n] = sum_k A[m, k] * W[n, k] + bias[n]  (A [M, K], W [N, K] row-major).
cudaError_t launch_rows_times_wt(const float* A, const float* W, const float* bias, int M, int K, int N, float* out,
                                 cudaStream_t s);

// ---- alpha-CROWN (k_alpha.cu) -----------------------------------------------------------
// Split constraints of one ReLU for the beta terms of the specification bound: the sign of each
// (centre, neuron) [B, n] (0 = free), the per-row multipliers [M, n], their Adam moments and the
// gradient output [M, n]. All null: no split constraint.
struct BetaRows {
    const signed char* split = nullptr;
    float* beta = nullptr;
    float* m1 = nullptr;
    float* m2 = nullptr;
    float* grad_out = nullptr;
};
cudaError_t launch_relax_alpha_rows(const float* H, long long M, int n, const float4* P, PassGeom pg,
                                    const float* alpha, float* Z, float* cst, cudaStream_t s, int with_bias = 1,
                                    int accumulate = 0, BetaRows bt = BetaRows{});
cudaError_t launch_concretize_grad(const float* lam, long long M, int n0, PassGeom pg, const float* centres, float eps,
                                   const float* cst, float* lb, float* G, cudaStream_t s);
cudaError_t launch_relax_grad_adam(float* G, const float* H, long long M, int n, const float4* P, PassGeom pg,
                                   float* alpha, float* grad_out, float* m1, float* m2, int adam_step, float lr,
                                   cudaStream_t s, BetaRows bt = BetaRows{});
// Split multipliers max(init, 0) (0 without init) and zero Adam moments.
cudaError_t launch_zero_moments(float* beta, float* m1, float* m2, long long count, cudaStream_t s,
                                const float* init = nullptr);
// Start slopes: P's lower slope per (centre, neuron), or init clamped to [0, 1] where init >= 0; zero moments.
cudaError_t launch_alpha_init(float* alpha, float* m1, float* m2, long long M, int n, const float4* P, PassGeom pg,
                              cudaStream_t s, const float* init = nullptr);
cudaError_t launch_best_update(float* best, const float* cur, long long M, int first, cudaStream_t s);
// P[i] = {1, 1, 0, 0}: a relaxation table that passes rows through unchanged (slopes 1, no intercept, no
// bias), so rows whose slopes were applied already can take the tensor-core contraction.
cudaError_t launch_identity_relax(float4* P, long long n, cudaStream_t s);

// ---- sound-in-fp32 mode (k_sound.cu) ----------------------------------------------------------
float gamma_up(long long K);
cudaError_t launch_sound_radius(float* zr, const float* S, const float* bias, long long total, long long n,
                                long long per_channel, float g, cudaStream_t s);
cudaError_t launch_abs_plus(const float* c, const float* r, long long total, float* T, cudaStream_t s);
cudaError_t launch_sound_relu(const float* c, const float* r, long long total, const signed char* split, float* oc,
                              float* orad, cudaStream_t s);
cudaError_t launch_sound_add(const float* c1, const float* r1, const float* c2, const float* r2, long long total,
                             float* oc, float* orad, cudaStream_t s);
cudaError_t launch_magnitude(const float* l, const float* u, long long total, int pos_only, float* M, cudaStream_t s);
cudaError_t launch_input_weight(const float* c, float eps, long long total, float g0, float* w, cudaStream_t s);
cudaError_t launch_affine_weight(float* w, const float* bias, const float* Mv, long long total, long long n,
                                 long long per_channel, float gQ, float gN, cudaStream_t s);
cudaError_t launch_relu_weight(const float4* P, const float* l, const float* u, long long total, float gN, float* w,
                               cudaStream_t s);
cudaError_t launch_scale_up(const float* M, long long total, float g, float* w, cudaStream_t s);
// cst[m] -= sum_j |row_j| w[b, j] (rows over one node, relaxed by rx when given), rounded down.
cudaError_t launch_row_budget(const RowRef& A, Relax rx, long long M, int n, PassGeom pg, const float* w, float* cst,
                              cudaStream_t s);

// ---- branch and bound (k_bab.cu) ------------------------------------------------------------
// Per subdomain: the neuron to split next (search-wide index, -1 if none is unstable), whether some
// pre-activation bound has l > u, the lowest row bound (max of two bound arrays when both are given)
// and the branching score of the chosen neuron.
struct BabPick {
    int best;
    int empty;
    float minlb;
    float score;
};
cudaError_t launch_bab_pick(const float* pre_lb, const float* pre_ub, int D, const long long* blk_off, const int* blk_n,
                            const int* gbase, int nl, const float* lb_a, const float* lb_b, int R, BabPick* out,
                            cudaStream_t s);
// dst[d, :] = src[:] for d < D (n floats per row).
cudaError_t launch_repeat_row(const float* src, long long n, int D, float* dst, cudaStream_t s);
// Branch-and-bound ascent states between a batch (alpha_out layout: per ReLU layer q a block [n, R, n_q] at
// n R gbase_q) and a pool of [R, sum_n] slots: scatter = 0 gathers batch <- pool[slot[i]] (-1 where slot[i] < 0),
// scatter = 1 writes pool[slot[i]] <- batch where slot[i] >= 0. meta_n / meta_g [device]: per layer n_q, gbase_q.
cudaError_t launch_bab_state(float* pool, const int* slot, int n, int R, long long sum_n, const int* meta_n,
                             const int* meta_g, int nl, float* batch, int scatter, cudaStream_t s);
// Row r's CROWN minimiser vertex of the box centre +/- eps: x[r, :] = centre - eps * sign(lam[r, :]), each
// coordinate rounded towards the centre so it stays inside the box. centre [n], lam and x [R, n], device.
cudaError_t launch_minimiser_points(const float* centre, const float* lam, float eps, long long n, int R, float* x,
                                    cudaStream_t s);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per (kernel,
// device, size); safe to call from several threads.
cudaError_t allow_dyn_smem(const void* func, int bytes);

// Records `msg` as this thread's vf_last_error() text and returns `code`.
int set_last_error(int code, const char* msg);

}  // namespace vf
