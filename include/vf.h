/*
 * vf.h -- C ABI of libvf.so: linear bound propagation (IBP + CROWN with alpha-slope
 * ReLU relaxation) for ReLU networks over an L-infinity input box, on one NVIDIA B200.
 *
 * Source page for the method: "Scaling Neural Network Verification with Tensor
 * Parallelism and Fully Sharded Data Parallelism" (gist.science summary of arXiv
 * 2606.09377). Its technical summary, section 1 (problem definition), states the task:
 * prove that a network satisfies a property for every input of a domain, using bound
 * propagation (IBP, CROWN, alpha-CROWN) whose weight matrices and linear relaxation
 * matrices A sit on one accelerator. Section 2.1 states that CROWN's backward pass
 * needs intermediate bounds to fix the ReLU relaxation slopes and that IBP can stand in
 * for them; sections 3 and 4.3 name the per-neuron alpha tensors (ReLU slopes).
 *
 * Conventions for every entry point:
 *  - Pointers marked [device] must be CUDA device memory of the current device;
 *    [host] pointers are host memory. All floating point data is fp32, row-major.
 *  - A network's activations are flattened in C order (channel, row, column).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Calls
 *    only enqueue work on it; outputs are valid once the stream reaches that point.
 *  - Return value: VF_OK (0) or a vf_status error code. On error nothing further is
 *    enqueued and vf_last_error() (per thread) describes the failure. No entry point
 *    aborts or throws across the ABI. Asynchronous CUDA faults surface as VF_ERR_CUDA
 *    on a later call or from vf_sync().
 *  - The caller owns every buffer it passes; the library owns only what vf_net_create
 *    allocates (device copies of the weights, derived tables and the workspace), which
 *    vf_net_destroy frees. A vf_net is not thread-safe: one call at a time per handle.
 */
#ifndef VF_H
#define VF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VF_OK = 0,
    VF_ERR_ARG = 1,         /* null pointer, bad enum, negative size */
    VF_ERR_SHAPE = 2,       /* inconsistent node shapes or sizes */
    VF_ERR_WORKSPACE = 3,   /* the workspace given to vf_net_create is too small for this call */
    VF_ERR_NONFINITE = 4,   /* NaN/Inf in eps, centres, C, weights or alpha */
    VF_ERR_CUDA = 5,        /* a CUDA runtime call or kernel failed */
    VF_ERR_TIMEOUT = 6,     /* a kernel gave up a bounded device wait (see vf_net_check) */
    VF_ERR_UNSUPPORTED = 7  /* valid request outside what this build implements */
} vf_status;

/* Node kinds. A network is an array of nodes in topological order: every `src`/`src2`
 * index is smaller than the node's own index; node 0 is the only VF_INPUT. */
typedef enum {
    VF_INPUT = 0,   /* shape (c, h, w); use (n, 1, 1) for a flat input */
    VF_DENSE = 1,   /* z = W h + b,  W [n_out, n_in], b [n_out]; h is src flattened */
    VF_CONV2D = 2,  /* cross-correlation, W [c_out, c_in, k, k], b [c_out], stride, pad (zeros) */
    VF_RELU = 3,    /* h = max(z, 0) of src */
    VF_ADD = 4      /* src + src2 (same shape) */
} vf_op;

typedef struct {
    int op;                /* vf_op */
    int src, src2;         /* producer node indices; src2 only for VF_ADD (else -1) */
    int c, h, w;           /* VF_INPUT only: input shape */
    int n_out;             /* VF_DENSE: output width; VF_CONV2D: output channels */
    int k, stride, pad;    /* VF_CONV2D only */
    const float* W;        /* [host or device] weights, layout above; copied at create */
    const float* b;        /* [host or device] bias; copied at create */
} vf_node_desc;

typedef struct vf_net vf_net;

/* Build a network handle on the current CUDA device. Weights are copied (host or
 * device source, detected per pointer) and checked for finiteness; derived tables
 * (|W|, [W; -W] start rows for intermediate passes) are built once here.
 * `workspace_bytes` is the device scratch the handle reserves for every later call
 * (allocated here, once); 0 selects 4 GiB. Calls whose fixed buffers do not fit return
 * VF_ERR_WORKSPACE; CROWN row blocks are otherwise sized to fit the workspace. */
int vf_net_create(const vf_node_desc* nodes /*[host] n_nodes*/, int n_nodes, size_t workspace_bytes,
                  vf_net** out_net /*[host]*/);
void vf_net_destroy(vf_net* net);

/* Number of neurons of node v (its flattened output size), or -1 if v is out of range. */
int vf_net_node_size(const vf_net* net, int v);
/* Sum of vf_net_node_size over all nodes: the row length of vf_ibp's bound arrays per centre block. */
long long vf_net_total_size(const vf_net* net);
/* Kind (VF_DENSE, ...), sources and size of node v; any output pointer may be NULL. VF_ERR_ARG if v is
 * out of range. */
int vf_net_node_info(const vf_net* net, int v, int* op, int* src, int* src2, long long* n);

/* IBP pass (technical summary, section 2.1: the cheap, sound interval substitute).
 * Box: centres[b] +/- eps (no clipping). For every node v, writes its interval bounds
 * into lb_all/ub_all at offset B * (sum of sizes of nodes before v), as a [B, n_v] block.
 * centres [device] [B, n0]; lb_all, ub_all [device] [B * vf_net_total_size(net)]. */
int vf_ibp(vf_net* net, const float* centres, int B, float eps, float* lb_all, float* ub_all, void* stream);

/* CROWN back-substitution of lower-bound rows (section 1: the linear relaxation
 * matrices A; section 2.1: the relaxation slopes come from intermediate bounds).
 * Rows: lambda0 [device] [B or 1, R, n_start] (centre stride lambda0_bstride elements;
 * 0 = one block shared by all centres) are coefficients over node `start_node`'s output.
 * Each ReLU reached uses the bounds of its source node found in lb_all/ub_all (layout of
 * vf_ibp) and alpha[v] [device] [B, n_v] for ReLU node v (NULL array or NULL entry =
 * adaptive slope 1 iff u >= -l; given slopes are clamped to [0, 1]).
 * Outputs: lambda_in [device] [B, R, n0] and const_out [device] [B, R] such that, for
 * every input x in any domain, row . node_start(x) >= lambda_in . x + const_out.
 * Upper bounds: pass -lambda0 and negate the result. */
int vf_crown_backward(vf_net* net, int start_node, const float* lambda0, int R, long long lambda0_bstride,
                      const float* lb_all, const float* ub_all, const float* const* alpha /*[host] n_nodes or NULL*/,
                      int B, float* lambda_in, float* const_out, void* stream);

/* Concretisation over the box centres[b] +/- eps (section 1: "all inputs in the domain"):
 * lb[b, r] = lambda[b, r, :] . centres[b, :] - eps * sum_i |lambda[b, r, i]| + cst[b, r].
 * lambda [device] [B, R, n0], cst [device] [B, R] (or NULL = 0), centres [device] [B, n0],
 * lb [device] [B, R]. No handle needed; no scratch memory. */
int vf_concretize(const float* lambda, const float* cst, const float* centres, float eps, int B, int R, int n0,
                  float* lb, void* stream);

typedef struct {
    /* [host] n_nodes entries or NULL. For each ReLU node v: 1 = refine the bounds of its
     * source by a CROWN pass (rows [I; -I]) before use, 0 = keep the IBP bounds (the IBP
     * substitution of section 2.1). NULL = CROWN for every ReLU. A source that is a single
     * affine node fed by the input already has exact IBP bounds and is never re-run. */
    const int* relu_crown;
    /* [host] n_nodes entries of [device] [B, n_v] slopes, or NULL (all adaptive). */
    const float* const* alpha;
    int both_sides;          /* 1: also compute upper bounds (rows -C) */
    int skip_finite_check;   /* 1: skip the device NaN/Inf scan of centres, C and alpha */
    /* [device] optional outputs [B * vf_net_total_size(net)] in the vf_ibp layout: the
     * bounds used for each ReLU source after refinement (other nodes: IBP bounds). */
    float* pre_lb;
    float* pre_ub;
    /* 1: the call never synchronises `stream` (no NaN/Inf scan, no unstable-neuron compaction;
     * the bounds are the same numbers), so it can be captured in a CUDA graph. */
    int no_host_sync;
    /* [host] n_nodes entries of [device] [B, n_v] signs, or NULL: branch-and-bound split constraints
     * (technical summary, sections 2.2 and 4.3: beta-CROWN with branch-and-bound). Each centre row b is
     * one subdomain of its box; for ReLU node v, +1 restricts it to the inputs where the ReLU's input
     * z_i >= 0, -1 to those where z_i <= 0, 0 leaves neuron i free. The IBP interval of a split neuron
     * is clamped to its sign (z >= 0: l = max(l, 0); z <= 0: u = min(u, 0), and the ReLU outputs 0),
     * which makes it stable, so its relaxation is exact on the subdomain. Every bound is then valid on
     * the subdomain only. A subdomain that holds no input shows up as some pre_lb > pre_ub.
     * vf_alpha_crown also optimises the split multipliers beta (see vf_alpha_beta_grad). */
    const signed char* const* split;
    /* 1: sound in fp32 (vf_verify_batch only; VF_ERR_UNSUPPORTED elsewhere). Every bound is widened by a
     * rigorous budget for its own rounding, so lb never exceeds the exact-arithmetic minimum over the
     * box (technical summary, section 4.2: soundness as a one-sided over-approximation). Interval ends
     * are rounded outwards with a gamma_K = K u / (1 - K u) term per dot product of K terms; the ReLU
     * intercept is rounded up; at every node a back-substituted row passes, its constant is lowered by
     * sum_i |row_i| w_i, with w that node's rounding weights (contraction gamma_K |W| M, bias, relaxation and
     * intercept terms, concretisation), rounded down. Contractions take the FFMA kernels (IEEE rounding),
     * not the tensor cores; receptive-field windows and the fused concretisation are off. */
    int sound;
    /* alpha-CROWN for the intermediate bounds (technical summary, sections 3 and 4.3: the per-neuron alpha
     * tensors; the reading is this library's): alpha_inter_iters > 0 runs, right after the CROWN pass of every
     * refined ReLU whose source p is a dense node, alpha_inter_iters Adam steps of size alpha_inter_lr (the
     * ascent of vf_alpha_crown: per-row slopes of every earlier ReLU, split multipliers where `split` is set)
     * on rows [e_j; -e_j] over p for the neurons j still unstable (l < 0 < u); l_j = max(l_j, best lower bound),
     * u_j = min(u_j, -best bound of -e_j), and the ReLU's relaxation is formed again before later layers use it.
     * Chain networks only (VF_ERR_UNSUPPORTED otherwise); reads unstable counts back (synchronises `stream`),
     * so not with no_host_sync; not with sound. 0 = off. */
    int alpha_inter_iters;
    float alpha_inter_lr;
    /* vf_alpha_crown only (NULL = off), [device], each one [B, R, n_v] block per ReLU node v in node order (the
     * layout of alpha_out): start slopes of the ascent (an entry < 0 starts from the adaptive slope; others are
     * clamped to [0, 1]), start split multipliers (clamped to >= 0; free neurons' entries do not enter the bound
     * and keep their start value), and the last iterate's split multipliers (0 for a layer without splits).
     * Adam's moments always start at zero. */
    const float* alpha_rows_init;
    const float* beta_rows_init;
    float* beta_rows_out;
} vf_opts;

/* Whole verification step (section 1): IBP, CROWN intermediate bounds, specification
 * pass, decision. C [device] [B or 1, R, n_L] over the last node (centre stride
 * C_bstride elements; 0 = shared). Outputs [device], [B, R] each:
 *   lb = max(IBP lower, CROWN lower); ub (both_sides only, else may be NULL) =
 *   min(IBP upper, CROWN upper); lb_ibp (or NULL) the IBP lower bound; verified (or NULL)
 *   1 iff lb > 0. opts [host] may be NULL (all defaults).
 * An intermediate pass only needs rows for the neurons whose IBP interval contains 0 (the
 * others keep their IBP bounds), so passes run over those neurons alone; sizing them reads
 * the per-centre counts back once per call, which synchronises `stream` (as does the finite
 * check unless skipped). VF_COMPACT=0 in the environment at vf_net_create keeps every pass
 * at rows [I; -I]. */
int vf_verify_batch(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                    const vf_opts* opts, float* lb, float* ub, float* lb_ibp, uint8_t* verified, void* stream);

/* alpha-CROWN (technical summary, section 1: alpha-CROWN; sections 3 and 4.3: the per-neuron alpha
 * tensors, i.e. the lower ReLU slopes): tightens the CROWN lower bounds of the specification rows by
 * optimising, separately for every (centre, row), the lower slope of each unstable ReLU (0 < u/(u-l) < 1)
 * within [0, 1], by `iters` steps of projected gradient ascent with Adam (betas 0.9, 0.999, step `lr`)
 * from the adaptive slopes. Intermediate bounds are computed as in vf_verify_batch (opts->relu_crown,
 * opts->alpha) and stay fixed. Any slope in [0, 1] gives a sound bound, so every iterate is sound.
 * Networks: any graph of this library whose last node is dense (chains of dense/convolution layers take
 * a fused path; residual graphs keep every node's coefficients); opts->both_sides returns
 * VF_ERR_UNSUPPORTED (pass -C for upper bounds).
 * Outputs [device]: lb [B, R] the best CROWN lower bound over the iterates (not intersected with IBP);
 * lb_start [B, R] (or NULL) the bound at the adaptive start; alpha_out (or NULL) the final slopes, one
 * [B, R, n_v] block per ReLU node v in node order. C [device] [B or 1, R, n_L] with centre stride C_bstride. */
int vf_alpha_crown(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                   const vf_opts* opts, int iters, float lr, float* lb, float* lb_start, float* alpha_out,
                   void* stream);

/* The specification rows' CROWN lower bounds at given per-row slopes alpha [device] (layout of
 * vf_alpha_crown's alpha_out; entries of stable neurons are ignored) and their gradient with respect to
 * those slopes, grad [device] (same layout; zero for stable neurons and where the coefficient over the
 * ReLU output is negative). Same networks and options as vf_alpha_crown. */
int vf_alpha_grad(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                  const vf_opts* opts, const float* alpha, float* lb, float* grad, void* stream);

/* vf_alpha_grad with split constraints (opts->split) and their multipliers (beta-CROWN, technical summary
 * sections 2.2 and 4.3; the Lagrangian reading): on a subdomain where s_i z_i >= 0, the bound of a row may
 * subtract beta_i s_i z_i for any beta_i >= 0, so the row's coefficient over z_i gains -beta_i s_i when
 * the back-substitution passes the ReLU. beta [device] and grad_beta [device] have alpha's layout (one
 * [B, R, n_v] block per ReLU node v); entries of free neurons are ignored (beta) and zero (grad_beta):
 * d lb / d beta_i = -s_i * (d lb / d coefficient over z_i). beta = NULL means all zero; grad_beta may be
 * NULL. vf_alpha_crown starts beta at 0 and takes the slopes' Adam step on it, projected to beta >= 0. */
int vf_alpha_beta_grad(vf_net* net, const float* centres, int B, float eps, const float* C, int R,
                       long long C_bstride, const vf_opts* opts, const float* alpha, const float* beta, float* lb,
                       float* grad_alpha, float* grad_beta, void* stream);

/* Branch and bound over ReLU splits for one property (technical summary, sections 2.2, 3 and 4.3:
 * complete verification by beta-CROWN with branch-and-bound; the page names the method only). The
 * property: every row of C [device] [R, n_L] is positive at every input of the box centre [device] [n0]
 * +/- eps. The search, run on the host with every bound computed on the device:
 *   1. candidate counterexamples, before any subdomain is bounded: the centre, then (when some row's bound
 *      over the whole box is <= 0) every row r's CROWN minimiser vertex x*_r = centre - eps * sign(lam_r),
 *      lam_r the row's back-substituted input coefficients (vf_crown_backward with the whole box's
 *      intermediate bounds), where the row's linear lower bound is attained; each coordinate is rounded
 *      towards the centre so every point lies inside the box. A row < 0 at one of these inputs is a
 *      counterexample (VF_BAB_FALSIFIED). The fp32 value there is only a rounded evaluation, so a negative
 *      row is confirmed by the sound-in-fp32 mode (vf_opts.sound, both sides, eps = 0): FALSIFIED needs that
 *      mode's upper bound, which the exact value on the fp32 weights cannot exceed, to be < 0 on some row; a
 *      row within rounding of 0 is not a counterexample and the search goes on;
 *   2. a subdomain's row bound is the larger of vf_verify_batch's and vf_alpha_crown's (alpha_iters Adam
 *      steps of size lr on the slopes and the split multipliers); the whole box is bounded first;
 *   3. each round takes the open subdomains with the lowest bound (ties: created first), at most
 *      batch / 2 of them, splits each on its neuron with the largest upper-relaxation intercept
 *      -u l / (u - l) over all ReLU layers (ties: first layer, lowest index) into z <= 0 and z >= 0, and
 *      bounds all children in one batch;
 *   4. a child closes when some pre-activation bound has l > u (it holds no input) or all its rows are
 *      > 0; a child with no unstable neuron left and a row <= 0 ends the search (VF_BAB_UNKNOWN), as does
 *      a spent budget of max_domains bounded subdomains;
 *   5. no open subdomain: VF_BAB_VERIFIED.
 * The call synchronises `stream` once per round. It allocates its own device buffers for the round
 * (batch subdomains) and uses the handle's workspace for the bounds. */
enum { VF_BAB_FALSIFIED = -1, VF_BAB_UNKNOWN = 0, VF_BAB_VERIFIED = 1 };
typedef struct {
    int max_domains;        /* budget of bounded subdomains, the whole box included (>= 1) */
    int batch;              /* subdomains bounded per round (even, >= 2) */
    int alpha_iters;        /* Adam steps per bound (0: vf_verify_batch's bound alone) */
    float lr;               /* Adam step size */
    const int* relu_crown;  /* as vf_opts.relu_crown */
    int* trace;             /* [host] or NULL: for every bounded subdomain in the order bounded (the whole box
                               first), the search-wide index of the neuron it would be split on (-1: none is
                               unstable); at most trace_cap entries are written, result->domains are bounded */
    int trace_cap;
    int alpha_inter_iters;  /* as vf_opts.alpha_inter_iters for every bound of the search (0: off): the subdomains'
                               intermediate bounds by alpha-CROWN, with the split multipliers of earlier layers */
    float alpha_inter_lr;
    int cold_start;         /* 0 (default): a child's ascent starts from its parent's last slopes and multipliers
                               (its new split's multiplier from 0), kept on the device for every open subdomain
                               while a pool of at most 1 GiB has room; 1: every ascent starts from the adaptive
                               slopes and zero multipliers */
} vf_bab_opts;
typedef struct {
    int status;             /* VF_BAB_VERIFIED, VF_BAB_FALSIFIED or VF_BAB_UNKNOWN */
    long long domains;      /* subdomains bounded, the whole box included (0 when falsified by step 1) */
    int rounds;             /* batched rounds after the whole box */
    int max_depth;          /* most splits in one bounded subdomain */
    float lb;               /* lowest row bound of the subdomains open at the end (+inf if none); when
                               falsified, the lowest fp32 row value at the candidate inputs that decided */
} vf_bab_result;
int vf_bab_verify(vf_net* net, const float* centre, float eps, const float* C, int R, const vf_bab_opts* opts,
                  vf_bab_result* result /*[host]*/, void* stream);

/* ABI self-description, for bindings that mirror the structs above (no device work): for struct `which`
 * (0 vf_node_desc, 1 vf_opts, 2 vf_bab_opts, 3 vf_bab_result) and `field` (index in declaration order, each
 * declarator counted once), writes the field's byte offset to *out; field = -1 writes the struct's size.
 * VF_ERR_ARG for an unknown struct or a field index past the last one. */
int vf_abi_layout(int which, int field, size_t* out);

/* The search of vf_bab_verify (steps 2-5) with a caller-supplied bound function, so other bounding
 * methods can drive it; vf_bab_verify is the centre check plus this search with the device bound function.
 * bound(user, n, ...) bounds n subdomains: subdomain i holds split_count[i] splits, listed from
 * split_offset[i] in split_neuron (search-wide neuron index: ReLU layers in node order, neurons in order)
 * and split_sign (+1: z >= 0, -1: z <= 0); it writes lb[i] (lowest row bound), branch[i] (the neuron to split
 * next, -1 if none is unstable) and empty[i] (1 if the subdomain holds no input), all [host], and returns
 * VF_OK or an error code, which ends the search with that code. A subdomain's splits are its parent's in
 * order, then the new one. Runs on the host only; the search itself touches no device. */
typedef int (*vf_bab_bound_fn)(void* user, int n, const int* split_offset, const int* split_count,
                               const int* split_neuron, const signed char* split_sign, float* lb, int* branch,
                               int* empty);
int vf_bab_search(vf_bab_bound_fn bound, void* user, int max_domains, int batch, vf_bab_result* result /*[host]*/);

/* Synchronise `stream` and report any pending asynchronous CUDA error. */
int vf_sync(void* stream);

/* Device-wide synchronising check of the handle's kernels: VF_ERR_TIMEOUT if any kernel launched
 * for `net` gave up a bounded wait (tensor-core pipeline barriers) since the last check, in which
 * case that call's outputs are not valid; clears the flag. */
int vf_net_check(vf_net* net);

/* Per-thread description of the last error (empty string if none). */
const char* vf_last_error(void);

/* Kernel timing, for benchmarks. While enabled, the library brackets each launch of a CROWN
 * back-substitution contraction with CUDA events on the launching stream. vf_profile_read
 * synchronises those events and returns, for one kind of contraction, the number of launches,
 * their summed device time in ms and their summed algorithmic flops (2*M*K*N for dense steps;
 * 2*M*n_in*C_out*k*k/stride^2 for whole-map convolutions, 2*M*(window positions on the map)*C_in*C_out*
 * k*k/stride^2 for receptive-field windows) since the last reset (reset != 0 clears all kinds). */
enum {
    VF_KERNEL_ALL = 0,
    VF_KERNEL_DENSE_TC = 1,
    VF_KERNEL_DENSE_FFMA = 2,
    VF_KERNEL_CONV = 3,
    VF_KERNEL_CONV_WIN = 4,
    VF_KERNEL_CONV_TC = 5, /* tensor-core implicit GEMM, whole maps and windows; flops as for windows */
    VF_KERNEL_DENSE_FWD_TC = 6, /* forward products on the tensor cores: the alpha gradient's G W^T + b (and with
                                   VF_FWD_TC=ibp at vf_net_create the IBP W c + b, |W| r); 2*M*K*N flops */
    VF_KERNEL_CONV_TC_PAD = 7  /* the tensor-core convolution on an input of fewer than 16 channels (padded to 16);
                                  flops of the real channels */
};
int vf_profile_enable(vf_net* net, int enable);
int vf_profile_read(vf_net* net, int kind, long long* launches, double* total_ms, double* flops, int reset);

/* Size, in floats, of the fixed scratch array used by vf_concretize_dense_noalloc (16 MiB). */
#define VF_NOALLOC_SCRATCH_FLOATS (1LL << 22)

/* Concretised back-substitution through one dense layer, for callers that cannot allocate device
 * memory: code whose device memory belongs to another allocator (a host framework's pool that forbids
 * cudaMalloc), code under a fixed device-memory budget, and code that must avoid the device-wide
 * synchronisation a cudaMalloc/cudaFree can cause. The page has no counterpart of this entry point; it
 * is the same arithmetic as vf_crown_backward from the layer followed by vf_concretize, without a handle
 * or workspace.
 *
 * Rows lambda [device] [B or 1, R, n_out] (centre stride lambda_bstride elements, 0 = shared) are
 * coefficients over z = W x + b, W [device] [n_out, n_in], b [device] [n_out]; x ranges over the box
 * centres[b] +/- eps, centres [device] [B, n_in]. Output lb [device] [B, R]:
 *   lb[b, r] = sum_i (lambda_r W)_i centres[b, i] - eps * sum_i |(lambda_r W)_i| + lambda_r . b.
 *
 * Scratch: a file-scope __device__ array of VF_NOALLOC_SCRATCH_FLOATS floats that every GPU loading the
 * library holds until exit; this call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine). It needs B*R*(1 + ceil(n_in / T)) floats with T = 64 for n_in <= 64, else 128; larger
 * requests return VF_ERR_WORKSPACE without launching anything (split the rows into several calls).
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, which may load
 * the library's device code), so make that first call before any stream capture. All calls share the
 * one array and it keeps the last call's contents (the row constants are cleared by each call): calls
 * whose execution overlaps on the GPU -- on different streams, or from different threads -- race and
 * must be serialised by the caller. The looked-up address is kept for the life of the process, so a
 * caller that resets a device (cudaDeviceReset) must not use this entry point on it afterwards.
 * lambda_bstride is 0 or at least R * n_out. Errors: VF_ERR_ARG, VF_ERR_NONFINITE (eps), VF_ERR_WORKSPACE,
 * VF_ERR_CUDA, described by vf_last_error(). */
int vf_concretize_dense_noalloc(const float* lambda, long long lambda_bstride, int R, const float* W, const float* b,
                                const float* centres, float eps, int B, int n_in, int n_out, float* lb, void* stream);

/* Number of kernel launches the library has enqueued on this handle since creation. */
long long vf_launch_count(const vf_net* net);

#ifdef __cplusplus
}
#endif
#endif /* VF_H */
