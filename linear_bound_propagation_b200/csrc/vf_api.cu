// Host side of libvf.so: the C ABI declared in include/vf.h, the network handle, the workspace
// arena and the executor that schedules the bound-propagation kernels on one stream.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism" (gist.science summary of arXiv 2606.09377), technical summary:
//   §1   the task (a property for every input of a domain) and the A matrices that must fit one
//        accelerator -- here they are streamed through a fixed workspace in row blocks;
//   §2.1 CROWN needs intermediate bounds for the ReLU relaxation slopes; IBP can replace them;
//   §3, §4.3 per-neuron alpha slopes.
//
// Execution of one verify call (everything enqueued on the caller's stream, no host sync
// except the optional finiteness scan):
//   1. IBP over every node (centre/radius form).
//   2. For each ReLU in topological order: optionally a CROWN pass over its source with rows
//      [I; -I] per centre (the first step through the source is the "identity trick": rows
//      become +-W rows with no contraction), then intersection with IBP, then the relaxation
//      parameters {lo, up, t} per neuron.
//   3. The specification pass (rows C, or [C; -C] for both sides) back to the input.
//   4. Decision: max(IBP, CROWN) lower bound, verified iff > 0.
// Passes are cut into row blocks sized to the workspace; rows are independent, so blocking
// changes nothing in any row's arithmetic.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "vf.h"
#include "vf_internal.cuh"
#include "vf_tc.cuh"

using namespace vf;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[1024];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

#define CU(call)                                                                                              \
    do {                                                                                                      \
        cudaError_t e_ = (call);                                                                              \
        if (e_ != cudaSuccess) return fail(VF_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));             \
    } while (0)

#define TRY(call)                       \
    do {                                \
        int r_ = (call);                \
        if (r_ != VF_OK) return r_;     \
    } while (0)

struct Node {
    int op = 0, src = -1, src2 = -1;
    int c = 0, h = 0, w = 0;
    long long n = 0;
    int k = 0, stride = 1, pad = 0;
    float* W = nullptr;
    float* Wabs = nullptr;
    float* b = nullptr;
    float* pmW = nullptr;  // dense only: [W; -W], the rows of the identity-trick first step
    float* WtHi = nullptr; // dense only: W^T [n_in, n_out] truncated to tf32 (3xTF32 head)
    float* WtLo = nullptr; // dense only: W^T - WtHi (3xTF32 remainder)
    float* WfHi = nullptr; // dense only: W [n_out, n_in] split the same way (forward products W c, G W^T)
    float* WfLo = nullptr;
    float* WaHi = nullptr; // dense only: |W| split: |WfHi| and |WfLo| (|w| truncates to |head|, remainder keeps sign)
    float* WaLo = nullptr;
    float* rowsum_abs = nullptr;  // dense only: sum_k |W[n, k]| (IBP radius of a layer fed by the input box)
    float* Wwin = nullptr;        // conv only: weights in the tap-major layout of the windowed kernel
    float* Wtc = nullptr;         // conv only: 3xTF32 operand images of the tensor-core kernel (or null)
    float* Wtn = nullptr;         // conv only: the same with the taps in N (k_back_conv_tcn.cu), or null
    WinWeights ww{nullptr, 0, 0, 4, 0};
    int consumers = 0;
};

}  // namespace

struct vf_net {
    std::vector<Node> nodes;
    int device = 0;
    int num_sms = 148;
    long long total = 0;
    char* ws = nullptr;
    size_t ws_bytes = 0;
    long long launches = 0;
    long long fail_at = 0;  // test hook: VF_TEST_FAIL_AT=<n> fails the n-th launch on the host
    // back-substitution through dense nodes: 0 (default) tensor cores where the shapes allow and the launch has at
    // least dense_tc_min_tiles output tiles (fewer tiles leave most SMs idle, where the K-split FFMA kernel is
    // faster), 1 FFMA only (VF_DENSE_KERNEL=ffma), 2 tensor cores whenever the shapes allow (VF_DENSE_KERNEL=tc)
    int dense_kernel = 0;
    long long dense_tc_min_tiles = 16;  // VF_DENSE_TC_MIN_TILES
    int* d_err = nullptr;   // device flag raised by a kernel whose bounded wait expired
    int tc_stall = 0;       // test hook: VF_TEST_TC_STALL=1 makes one tensor-core launch time out
    int windows = 1;        // receptive-field windows in passes that start at a convolution (VF_CONV_WINDOWS=0: off)
    // whole-map rows through the one-warp-per-row windowed kernel: 0 never (VF_CONV_KERNEL=tile), 1 whenever
    // its staging fits (VF_CONV_KERNEL=warp), 2 (default) when it fits with a full CTA and staged weights
    int conv_whole_warp = 2;
    int conv_win_per_position = 0;  // windowed rows without position blocking (VF_CONV_WIN_KERNEL=1)
    int compact = 1;        // intermediate passes over IBP-unstable neurons only (VF_COMPACT=0: off)
    int conv_tc = 1;        // convolution steps on the tensor cores where the shapes allow (VF_CONV_TC=0: off)
    int conv_tcn = 0;       // ... with the taps-in-N kernel where its shapes allow (VF_CONV_TC=tapn; measured slower)
    int call_sound = 0;     // set for the duration of a vf_opts.sound call: contractions take FFMA kernels
    // forward products of the alpha ascent (G W^T + b) on the tensor cores: 0 never (VF_FWD_TC=0), 1 (default) when
    // the product has at least kFwdTcMinTiles output tiles, 2 whenever the shapes allow (VF_FWD_TC=all); 3 also the
    // IBP products W c + b, |W| r (VF_FWD_TC=ibp; less accurate on deep wide networks, see run_ibp)
    int fwd_tc = 1;
    float4* ident_row = nullptr;  // identity relaxation row {1, 1, 0, 0} x (largest node size), for forward products
    bool prof = false;
    std::vector<cudaEvent_t> ev_free;
    struct Timed {
        cudaEvent_t e0, e1;
        int kind;
        double flops;
    };
    std::vector<Timed> ev_used;
    double prof_flops[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    long long prof_launches[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    double prof_ms[8] = {0, 0, 0, 0, 0, 0, 0, 0};
};

namespace {

ConvGeom conv_geom(const vf_net* net, const Node& nd) {
    const Node& s = net->nodes[nd.src];
    ConvGeom g;
    g.ci = s.c;
    g.h = s.h;
    g.w = s.w;
    g.co = nd.c;
    g.ho = nd.h;
    g.wo = nd.w;
    g.k = nd.k;
    g.stride = nd.stride;
    g.pad = nd.pad;
    return g;
}

// Counts launches and turns launch errors into VF_ERR_CUDA.
int launched(vf_net* net, cudaError_t e, const char* what) {
    net->launches++;
    if (e != cudaSuccess) return fail(VF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return VF_OK;
}

// Test hook: with VF_TEST_FAIL_AT=<n> in the environment at vf_net_create, the n-th launch of
// the handle is not issued and the call fails with VF_ERR_CUDA (host-side fault injection).
#define LAUNCH(net, expr)                                                                           \
    do {                                                                                            \
        if ((net)->fail_at > 0 && (net)->launches + 1 == (net)->fail_at) {                          \
            (net)->launches++;                                                                      \
            return fail(VF_ERR_CUDA, "injected failure before launch %lld", (net)->launches);       \
        }                                                                                           \
        TRY(launched((net), (expr), #expr));                                                        \
    } while (0)

cudaEvent_t take_event(vf_net* net) {
    if (!net->ev_free.empty()) {
        cudaEvent_t e = net->ev_free.back();
        net->ev_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

struct Arena {
    char* base;
    size_t cap, off = 0;
    template <typename T>
    T* take(size_t count) {
        size_t o = (off + 255) & ~size_t(255);
        size_t bytes = count * sizeof(T);
        if (o + bytes > cap) return nullptr;
        off = o + bytes;
        return reinterpret_cast<T*>(base + o);
    }
    size_t left() const {
        size_t o = (off + 255) & ~size_t(255);
        return o >= cap ? 0 : cap - o;
    }
};

// -------------------------------------------------------------------------------------------
// Walker: back-substitutes one row block of one pass through the node graph.
// -------------------------------------------------------------------------------------------
enum EntryKind { E_NONE = 0, E_BUF = 1, E_VIRT = 2, E_IDENT = 3 };

struct Entry {
    int kind = E_NONE;
    int buf = -1;  // E_BUF: pool index
    RowRef ref{nullptr, 0, 0, kHugeRows, 0};
    Relax rx{nullptr, 0};
    bool windowed = false;  // rows held as a receptive-field window `win` of the node's map
    Win win{0, 0, 0, 0, 0, 0, 0};
};

// Receptive-field windows (rows of a pass that starts at a convolution, see k_win.cu).
Win full_win(const Node& nd) { return Win{nd.c, nd.h, nd.w, 0, 0, 0, 0}; }
// The 1 x 1 window at the start position: identity start rows on a node shaped like the start node.
Win ident_win(const Node& nd) { return Win{nd.c, 1, 1, 1, 0, 1, 0}; }
long long win_len(const Win& w) { return (long long)w.C * w.hh * w.hw; }
bool win_eq(const Win& a, const Win& b) {
    return a.C == b.C && a.hh == b.hh && a.hw == b.hw && a.ay == b.ay && a.by == b.by && a.ax == b.ax && a.bx == b.bx;
}
// Field over a convolution's input of rows in window `wa` over its output.
Win win_back(const Win& wa, const ConvGeom& g) {
    return Win{g.ci,
               g.stride * (wa.hh - 1) + g.k,
               g.stride * (wa.hw - 1) + g.k,
               g.stride * wa.ay,
               g.stride * wa.by - g.pad,
               g.stride * wa.ax,
               g.stride * wa.bx - g.pad};
}
// A window is kept only while it holds at most half of the node's map.
bool win_small(const Win& w, const Node& nd) { return nd.h > 1 && 2 * win_len(w) <= nd.n; }
// Smallest window containing both (same channel count and origin slopes), else false.
bool win_union(const Win& a, const Win& b, Win* u) {
    if (a.C != b.C || a.ay != b.ay || a.ax != b.ax) return false;
    const int by = std::min(a.by, b.by), bx = std::min(a.bx, b.bx);
    *u = Win{a.C, std::max(a.by + a.hh, b.by + b.hh) - by, std::max(a.bx + a.hw, b.bx + b.hw) - bx, a.ay, by, a.ax, bx};
    return true;
}

// Dense back-substitution of M rows onto a node of N neurons on the tensor cores (the kernel's own shape
// checks aside): not in FFMA-only or sound calls, and by default only when the launch has enough output tiles.
bool back_tc_ok(const vf_net* net, long long M, int N) {
    if (net->dense_kernel == 1 || net->call_sound) return false;
    return net->dense_kernel == 2 || ((M + 127) / 128) * dense_back_tc_tiles_n(N) >= net->dense_tc_min_tiles;
}

struct Walker {
    vf_net* net;
    cudaStream_t s;
    bool dry;                 // only count buffers
    long long M;              // rows in this block
    PassGeom pg;
    float* cst;               // [M]
    float* part;              // [tiles, M] partials of a fused concretisation
    int part_tiles = 0;       // set when the fused concretisation ran
    std::vector<float*> bufs;
    std::vector<int> ref;
    long long ld_buf;
    int live = 0, max_live = 0;
    const float* centres = nullptr;
    float eps = 0.f;
    long long n_centres = 0;  // rows of the relaxation tables
    float* ext_in = nullptr;  // vf_crown_backward: rows over the input go here ([M, n0], ld n0)
    bool ext_written = false;
    const std::vector<const float4*>* relax;  // per node: relaxation params of ReLU nodes
    std::vector<Entry> pend;
    bool win_on = false;      // rows may be held as receptive-field windows (pass starts at a convolution)
    bool compact = false;     // identity-trick pass over the listed unstable neurons only (pg.idx)
    PassStart ps{1, 1, 1};    // the pass's start node
    long long max_len = 0;    // longest row a pool buffer has held
    const std::vector<float*>* sw = nullptr;  // sound mode: per-node rounding weights [B, n_v]

    int alloc_buf(int* out, long long len) {
        max_len = std::max(max_len, len);
        if (!dry && len > ld_buf) return fail(VF_ERR_WORKSPACE, "row of %lld floats exceeds the row buffers", len);
        for (size_t i = 0; i < ref.size(); ++i)
            if (ref[i] == 0) {
                ref[i] = 1;
                live++;
                max_live = std::max(max_live, live);
                *out = (int)i;
                return VF_OK;
            }
        if (dry) {
            ref.push_back(1);
            bufs.push_back(nullptr);
            live++;
            max_live = std::max(max_live, live);
            *out = (int)ref.size() - 1;
            return VF_OK;
        }
        return fail(VF_ERR_WORKSPACE, "row-block buffer pool exhausted");
    }
    void release(Entry& e) {
        if (e.kind == E_BUF && --ref[e.buf] == 0) live--;
        e = Entry();
    }
    RowRef local(int b) const { return RowRef{dry ? nullptr : bufs[b], 0, ld_buf, kHugeRows, 0}; }
    Entry buf_entry(int b) const {
        Entry e;
        e.kind = E_BUF;
        e.buf = b;
        e.ref = local(b);
        return e;
    }

    // Make pend[v] a plain (unrelaxed, unshared) buffer so contributions can be added to it, held as
    // window *want (which contains the entry's window), or as the whole map when want is null.
    int make_plain(int v, int* out, const Win* want = nullptr) {
        Entry& e = pend[v];
        const Node& nd = net->nodes[v];
        const long long n = nd.n;
        const bool same = want ? (e.windowed && win_eq(e.win, *want)) : !e.windowed;
        if (e.kind == E_BUF && same && ref[e.buf] == 1) {
            if (e.rx.P != nullptr) {  // relax in place
                if (!dry) {
                    if (e.windowed)
                        LAUNCH(net, launch_rewin_rows(e.ref, e.rx, M, nd.c, nd.h, nd.w, pg, ps, e.win, e.win,
                                                      bufs[e.buf], ld_buf, 0, cst, s));
                    else
                        LAUNCH(net, launch_relax_rows(e.ref, e.rx, M, (int)n, pg, bufs[e.buf], ld_buf, 0, cst, s));
                }
                e.rx = Relax{nullptr, 0};
            }
            *out = e.buf;
            return VF_OK;
        }
        int nb;
        TRY(alloc_buf(&nb, want ? win_len(*want) : n));
        if (!dry) {
            if (e.kind == E_IDENT && want != nullptr)
                LAUNCH(net, launch_ident_rows_win(bufs[nb], ld_buf, M, pg, ps, *want, 0, s));
            else if (e.kind == E_IDENT)
                LAUNCH(net, launch_ident_rows(bufs[nb], ld_buf, M, pg, n, 0, s));
            else if (!e.windowed && want == nullptr)
                LAUNCH(net, launch_relax_rows(e.ref, e.rx, M, (int)n, pg, bufs[nb], ld_buf, 0, cst, s));
            else
                LAUNCH(net, launch_rewin_rows(e.ref, e.rx, M, nd.c, nd.h, nd.w, pg, ps, e.windowed ? e.win : full_win(nd),
                                              want ? *want : full_win(nd), bufs[nb], ld_buf, 0, cst, s));
        }
        release(e);
        pend[v] = buf_entry(nb);
        if (want != nullptr) {
            pend[v].windowed = true;
            pend[v].win = *want;
        }
        *out = nb;
        return VF_OK;
    }

    // Window of entry e at node v; false for whole-map rows.
    bool entry_win(int v, const Entry& e, Win* w) const {
        if (e.windowed) {
            *w = e.win;
            return true;
        }
        if (e.kind == E_IDENT && win_on && e.rx.P == nullptr && win_small(ident_win(net->nodes[v]), net->nodes[v])) {
            *w = ident_win(net->nodes[v]);
            return true;
        }
        return false;
    }

    // The window that holds both pend[v] and rows in window x (null: the whole map).
    bool merged_win(int v, const Win* x, Win* u) const {
        Win ew;
        return x != nullptr && entry_win(v, pend[v], &ew) && win_union(ew, *x, u) && win_small(*u, net->nodes[v]);
    }

    // pend[v] += x (x is consumed).
    int add_into(int v, Entry x) {
        if (pend[v].kind == E_NONE) {
            pend[v] = x;
            return VF_OK;
        }
        const Node& nd = net->nodes[v];
        const long long n = nd.n;
        Win xw, u;
        const bool xwin = entry_win(v, x, &xw);
        const bool wu = merged_win(v, xwin ? &xw : nullptr, &u);
        int b;
        TRY(make_plain(v, &b, wu ? &u : nullptr));
        if (!dry) {
            if (x.kind == E_IDENT && wu)
                LAUNCH(net, launch_ident_rows_win(bufs[b], ld_buf, M, pg, ps, u, 1, s));
            else if (x.kind == E_IDENT)
                LAUNCH(net, launch_ident_rows(bufs[b], ld_buf, M, pg, n, 1, s));
            else if (!x.windowed && !wu)
                LAUNCH(net, launch_relax_rows(x.ref, x.rx, M, (int)n, pg, bufs[b], ld_buf, 1, cst, s));
            else
                LAUNCH(net, launch_rewin_rows(x.ref, x.rx, M, nd.c, nd.h, nd.w, pg, ps, x.windowed ? x.win : full_win(nd),
                                              wu ? u : full_win(nd), bufs[b], ld_buf, 1, cst, s));
        }
        release(x);
        return VF_OK;
    }

    // Where an affine node's back-substituted rows over its source go. nat: the window the rows
    // occupy (null: the whole map); *dst receives the window of the destination (the whole map when
    // the entry there is not windowed).
    int target(int src, float** out, long long* ld, int* mode, const Win* nat = nullptr, Win* dst = nullptr) {
        const Node& sn = net->nodes[src];
        if (dst != nullptr) *dst = full_win(sn);
        if (src == 0 && ext_in != nullptr && pend[0].kind == E_NONE) {
            *out = ext_in;
            *ld = net->nodes[0].n;
            *mode = ext_written ? OUT_ACCUM : OUT_STORE;
            ext_written = true;
            return VF_OK;
        }
        if (pend[src].kind == E_NONE) {
            const bool wnd = nat != nullptr && win_small(*nat, sn);
            int nb;
            TRY(alloc_buf(&nb, wnd ? win_len(*nat) : sn.n));
            pend[src] = buf_entry(nb);
            if (wnd) {
                pend[src].windowed = true;
                pend[src].win = *nat;
                if (dst != nullptr) *dst = *nat;
            }
            *out = dry ? nullptr : bufs[nb];
            *ld = ld_buf;
            *mode = OUT_STORE;
            return VF_OK;
        }
        Win u;
        const bool wu = merged_win(src, nat, &u);
        int b;
        TRY(make_plain(src, &b, wu ? &u : nullptr));
        if (wu && dst != nullptr) *dst = u;
        *out = dry ? nullptr : bufs[b];
        *ld = ld_buf;
        *mode = OUT_ACCUM;
        return VF_OK;
    }

    void prof_begin(cudaEvent_t* e0) {
        if (net->prof && !dry) {
            *e0 = take_event(net);
            cudaEventRecord(*e0, s);
        }
    }
    void prof_end(cudaEvent_t e0, int kind, double flops) {
        if (net->prof && !dry) {
            cudaEvent_t e1 = take_event(net);
            cudaEventRecord(e1, s);
            net->ev_used.push_back({e0, e1, kind, flops});
        }
    }

    int process(int v) {
        Entry e = pend[v];
        pend[v] = Entry();
        if (e.kind == E_NONE) return VF_OK;
        const Node& nd = net->nodes[v];
        // sound mode: the rounding budget of these rows at this node (identity starts are exact)
        if (sw != nullptr && !dry && e.kind != E_IDENT && (*sw)[v] != nullptr)
            LAUNCH(net, launch_row_budget(e.ref, e.rx, M, (int)nd.n, pg, (*sw)[v], cst, s));
        switch (nd.op) {
            case VF_INPUT: {
                if (e.kind == E_IDENT || e.rx.P != nullptr || e.windowed) {
                    pend[0] = e;
                    int b;
                    TRY(make_plain(0, &b));
                    e = pend[0];
                    pend[0] = Entry();
                }
                if (ext_in != nullptr) {
                    if (!dry)
                        LAUNCH(net, launch_relax_rows(e.ref, Relax{nullptr, 0}, M, (int)nd.n, pg, ext_in, nd.n,
                                                      ext_written ? 1 : 0, nullptr, s));
                    ext_written = true;
                } else if (!dry) {
                    LAUNCH(net, launch_concretize_rows(e.ref, M, (int)nd.n, pg, centres, eps, cst, s));
                }
                release(e);
                return VF_OK;
            }
            case VF_RELU: {
                if (e.kind == E_IDENT || e.rx.P != nullptr) {
                    Win ew;
                    const bool wnd = entry_win(v, e, &ew);
                    pend[v] = e;
                    int b;
                    TRY(make_plain(v, &b, wnd ? &ew : nullptr));
                    e = pend[v];
                    pend[v] = Entry();
                }
                e.rx = Relax{(*relax)[v], 1};
                return add_into(nd.src, e);
            }
            case VF_ADD: {
                Entry y = e;
                y.rx.count_const = 0;
                if (e.kind == E_BUF) ref[e.buf]++;
                TRY(add_into(nd.src, e));
                return add_into(nd.src2, y);
            }
            case VF_DENSE: {
                const Node& sn = net->nodes[nd.src];
                if (e.windowed) {  // dense rows span the whole map
                    pend[v] = e;
                    int b;
                    TRY(make_plain(v, &b));
                    e = pend[v];
                    pend[v] = Entry();
                }
                if (e.kind == E_IDENT) {
                    if (!dry) LAUNCH(net, launch_cst_identity_bias(cst, M, pg, nd.b, nd.n, 1, s));
                    if (compact) {  // the listed neurons' rows +-W[j] are gathered into a buffer
                        int nb;
                        TRY(alloc_buf(&nb, sn.n));
                        if (!dry) LAUNCH(net, launch_gather_start_rows(bufs[nb], ld_buf, M, pg, nd.W, nd.n, sn.n, s));
                        return add_into(nd.src, buf_entry(nb));
                    }
                    Entry x;
                    x.kind = E_VIRT;
                    x.ref = RowRef{nd.pmW, 0, sn.n, 2 * nd.n, pg.pass_m0};
                    return add_into(nd.src, x);
                }
                const bool fuse = (nd.src == 0 && ext_in == nullptr && net->nodes[0].consumers == 1 && sw == nullptr &&
                                   pend[0].kind == E_NONE);
                float* out = nullptr;
                long long ld = 0;
                int mode = OUT_CONCRETIZE;
                if (!fuse) TRY(target(nd.src, &out, &ld, &mode));
                const bool tc = back_tc_ok(net, M, (int)sn.n) && nd.WtHi != nullptr &&
                                dense_back_tc_supported(e.ref, e.rx, M, (int)nd.n, (int)sn.n, pg);
                if (fuse) part_tiles = tc ? dense_back_tc_tiles_n((int)sn.n) : dense_back_tiles_n((int)sn.n);
                if (!dry) {
                    cudaEvent_t e0 = nullptr;
                    prof_begin(&e0);
                    if (tc) {
                        LAUNCH(net, launch_dense_back_tc(e.ref, e.rx, nd.WtHi, nd.WtLo, n_centres, M, (int)nd.n, (int)sn.n, pg,
                                                         mode, out, ld, cst, centres, eps, part, net->d_err,
                                                         net->tc_stall, s));
                        net->tc_stall = 0;  // the test hook withholds one copy, once
                    } else
                        LAUNCH(net, launch_dense_back(e.ref, e.rx, nd.W, nd.b, M, (int)nd.n, (int)sn.n, pg, mode, out,
                                                      ld, cst, centres, eps, part, s));
                    prof_end(e0, tc ? VF_KERNEL_DENSE_TC : VF_KERNEL_DENSE_FFMA, 2.0 * (double)M * (double)nd.n * (double)sn.n);
                }
                release(e);
                return VF_OK;
            }
            case VF_CONV2D: {
                const ConvGeom g = conv_geom(net, nd);
                const Node& sn = net->nodes[nd.src];
                if (e.kind == E_IDENT) {
                    if (!dry)
                        LAUNCH(net, launch_cst_identity_bias(cst, M, pg, nd.b, nd.n, (long long)nd.h * nd.w, s));
                    float* out = nullptr;
                    long long ld = 0;
                    int mode = OUT_STORE;
                    if (win_on) {  // the k x k field of each start neuron
                        const Win nat{g.ci, g.k, g.k, g.stride, -g.pad, g.stride, -g.pad};
                        Win dst;
                        TRY(target(nd.src, &out, &ld, &mode, &nat, &dst));
                        if (!dry)
                            LAUNCH(net, launch_conv_start_rows_win(out, ld, M, pg, ps, nd.W, g, dst,
                                                                   mode == OUT_ACCUM ? 1 : 0, s));
                        return VF_OK;
                    }
                    TRY(target(nd.src, &out, &ld, &mode));
                    if (!dry)
                        LAUNCH(net, launch_conv_start_rows(out, ld, M, pg, nd.W, g, mode == OUT_ACCUM ? 1 : 0, s));
                    return VF_OK;
                }
                const bool fuse_in = (nd.src == 0 && ext_in == nullptr && net->nodes[0].consumers == 1 &&
                                      sw == nullptr && pend[0].kind == E_NONE);
                const Win wa_tc = e.windowed ? e.win : full_win(nd);
                const bool tcn = net->conv_tc && net->conv_tcn && !net->call_sound && sw == nullptr &&
                                 nd.Wtn != nullptr && conv_back_tcn_supported(g, wa_tc, full_win(sn), OUT_CONCRETIZE);
                if (tcn || (net->conv_tc && !net->call_sound && sw == nullptr && nd.Wtc != nullptr &&
                            conv_back_tc_supported(g, wa_tc, full_win(sn), OUT_CONCRETIZE))) {
                    // tensor-core implicit GEMM, for whole-map and windowed rows alike
                    float* out = nullptr;
                    long long ld = 0;
                    int mode = OUT_CONCRETIZE;
                    Win dst = full_win(sn);
                    if (!fuse_in) {
                        if (e.windowed) {
                            const Win nat = win_back(e.win, g);
                            dst = win_small(nat, sn) ? nat : full_win(sn);
                            TRY(target(nd.src, &out, &ld, &mode, &nat, &dst));
                        } else {
                            TRY(target(nd.src, &out, &ld, &mode));
                        }
                    }
                    if (!dry) {
                        if (mode == OUT_STORE && !conv_back_tc_covers(g, wa_tc, dst))
                            CU(cudaMemset2DAsync(out, sizeof(float) * ld, 0, sizeof(float) * win_len(dst), M, s));
                        cudaEvent_t e0 = nullptr;
                        prof_begin(&e0);
                        if (tcn)
                            LAUNCH(net, launch_conv_back_tcn(e.ref, e.rx, nd.Wtn, nd.b, M, g, pg, ps, wa_tc, dst, mode,
                                                             out, ld, cst, centres, eps, net->d_err, net->num_sms, s));
                        else
                            LAUNCH(net, launch_conv_back_tc(e.ref, e.rx, nd.Wtc, nd.b, M, g, pg, ps, wa_tc, dst, mode,
                                                            out, ld, cst, centres, eps, net->d_err, net->num_sms, s));
                        const Win nat = win_back(wa_tc, g);
                        const double pos = (double)std::min<long long>((long long)nat.hh * nat.hw, (long long)g.h * g.w);
                        prof_end(e0, g.ci % 16 == 0 ? VF_KERNEL_CONV_TC : VF_KERNEL_CONV_TC_PAD,
                                 2.0 * (double)M * pos * g.ci * g.co * g.k * g.k / ((double)g.stride * g.stride));
                    }
                    release(e);
                    return VF_OK;
                }
                WinLaunch wl;
                if (!e.windowed && e.kind != E_IDENT && net->conv_whole_warp &&
                    conv_back_win_plan(g, nd.ww, full_win(nd), &wl) &&
                    (net->conv_whole_warp == 1 ||
                     conv_back_win_whole_map_fits(g, nd.ww, full_win(nd), full_win(sn)))) {  // rows as one full window
                    e.windowed = true;
                    e.win = full_win(nd);
                }
                if (e.windowed && !conv_back_win_plan(g, nd.ww, e.win, &wl)) {  // staging too large
                    pend[v] = e;
                    int b;
                    TRY(make_plain(v, &b));
                    e = pend[v];
                    pend[v] = Entry();
                }
                const bool fuse = (nd.src == 0 && ext_in == nullptr && net->nodes[0].consumers == 1 && sw == nullptr &&
                                   pend[0].kind == E_NONE);
                float* out = nullptr;
                long long ld = 0;
                int mode = OUT_CONCRETIZE;
                if (e.windowed) {
                    const Win nat = win_back(e.win, g);
                    Win dst = win_small(nat, sn) ? nat : full_win(sn);
                    if (!fuse) TRY(target(nd.src, &out, &ld, &mode, &nat, &dst));
                    if (!dry) {
                        cudaEvent_t e0 = nullptr;
                        prof_begin(&e0);
                        LAUNCH(net, launch_conv_back_win(e.ref, e.rx, nd.ww, nd.b, M, g, pg, ps, e.win, dst, mode, out, ld,
                                                         cst, centres, eps, s));
                        const double pos = (double)std::min<long long>((long long)dst.hh * dst.hw, (long long)g.h * g.w);
                        prof_end(e0, VF_KERNEL_CONV_WIN, 2.0 * (double)M * pos * g.ci * g.co * g.k * g.k /
                                                         ((double)g.stride * g.stride));
                    }
                    release(e);
                    return VF_OK;
                }
                if (!fuse) TRY(target(nd.src, &out, &ld, &mode));
                if (fuse) part_tiles = conv_back_tiles(g);
                if (!dry) {
                    cudaEvent_t e0 = nullptr;
                    prof_begin(&e0);
                    LAUNCH(net, launch_conv_back(e.ref, e.rx, nd.W, nd.b, M, g, pg, mode, out, ld, part, centres, eps,
                                                 net->num_sms, s));
                    prof_end(e0, VF_KERNEL_CONV, 2.0 * (double)M * (double)net->nodes[nd.src].n * (double)g.co * g.k *
                                                     g.k / ((double)g.stride * g.stride));
                    if (!fuse) LAUNCH(net, launch_add_partials(cst, part, conv_back_tiles(g), M, s));
                }
                release(e);
                return VF_OK;
            }
        }
        return fail(VF_ERR_ARG, "bad node kind");
    }

    // Back-substitute from node `start` whose rows are `init`, down to the input.
    int run(int start, Entry init) {
        pend.assign(net->nodes.size(), Entry());
        part_tiles = 0;
        ext_written = false;
        live = 0;
        for (auto& r : ref) r = 0;
        if (!dry) CU(cudaMemsetAsync(cst, 0, sizeof(float) * M, s));
        pend[start] = init;
        for (int v = start; v >= 0; --v) TRY(process(v));
        return VF_OK;
    }
};

long long max_node_size(const vf_net* net, bool include_input) {
    long long m = 1;
    for (size_t v = include_input ? 0 : 1; v < net->nodes.size(); ++v) m = std::max(m, net->nodes[v].n);
    return m;
}

// A source whose IBP bounds are already the exact range: the input itself, or one affine node
// fed directly by the input (its interval c +- |W| eps is attained coordinate by coordinate).
bool exact_source(const vf_net* net, int p) {
    const Node& nd = net->nodes[p];
    return p == 0 || ((nd.op == VF_DENSE || nd.op == VF_CONV2D) && nd.src == 0);
}

// Rows over the input are held in a buffer unless its only consumer is one affine node, whose
// contraction then writes (or concretises) them directly.
bool input_buffered(const vf_net* net) {
    if (net->nodes[0].consumers != 1) return true;
    for (size_t v = 1; v < net->nodes.size(); ++v)
        if (net->nodes[v].src == 0 || net->nodes[v].src2 == 0)
            return !(net->nodes[v].op == VF_DENSE || net->nodes[v].op == VF_CONV2D);
    return true;
}

// Buffers a pass needs at once and the longest row they hold, by a dry run of the walker.
int pool_size(vf_net* net, int start, Entry init, const std::vector<const float4*>* relax, bool ext, bool win_on,
              bool compact, int* nb, long long* max_len, const std::vector<float*>* sw = nullptr) {
    Walker w;
    w.net = net;
    w.s = nullptr;
    w.dry = true;
    w.M = 1;
    w.pg = PassGeom{0, 1};
    w.cst = nullptr;
    w.part = nullptr;
    w.ld_buf = 1;
    w.relax = relax;
    w.win_on = win_on;
    w.compact = compact;
    w.sw = sw;  // the same fusion decisions as the real walk
    float dummy = 0.f;
    w.ext_in = ext ? &dummy : nullptr;
    TRY(w.run(start, init));
    *nb = w.max_live;
    *max_len = w.max_len;
    return VF_OK;
}

// Fewest 128 x (<= 256) output tiles for which a forward product takes the tensor-core kernel by default: it runs
// one persistent CTA per tile, so a product of a few tiles (the IBP of 1024 centres through 256 neurons: 8 tiles;
// the ascent of 64 branch-and-bound subdomains: 5) leaves most SMs idle and is slower than the FFMA kernel's 64 x 64
// tiles (measured on the 784-256x3-10 network). Products measured faster on the tensor cores had 72 tiles (the
// alpha ascent at 1024 centres) and 128 (the IBP of the 3072-1024x8-100 network at 4096 centres); the threshold
// sits between the two groups.
constexpr long long kFwdTcMinTiles = 32;

bool fwd_tc_ok(const vf_net* net, const Node& nd, const float* A, long long M, int K) {
    const int N = (int)nd.n;
    if (net->dense_kernel == 1 || net->fwd_tc == 0 || net->call_sound || nd.WfHi == nullptr) return false;
    if (!dense_fwd_tc_supported(A, M, K, N)) return false;
    return net->fwd_tc >= 2 || ((M + 127) / 128) * dense_back_tc_tiles_n(N) >= kFwdTcMinTiles;
}

// out [M, N] = A [M, K] W^T + bias (absw: A |W|^T, no bias) for dense node nd: the tensor-core kernel where
// fwd_tc_ok (profiled as VF_KERNEL_DENSE_FWD_TC), else the FFMA kernel.
int fwd_product(vf_net* net, const Node& nd, const float* A, long long M, int K, bool absw, const float* bias,
                float* out, cudaStream_t s) {
    const int N = (int)nd.n;
    if (fwd_tc_ok(net, nd, A, M, K)) {
        cudaEvent_t e0 = nullptr;
        if (net->prof) {
            e0 = take_event(net);
            cudaEventRecord(e0, s);
        }
        LAUNCH(net, launch_dense_fwd_tc(A, M, K, N, absw ? nd.WaHi : nd.WfHi, absw ? nd.WaLo : nd.WfLo,
                                        absw ? nullptr : bias, net->ident_row, out, net->d_err, s));
        if (net->prof) {
            cudaEvent_t e1 = take_event(net);
            cudaEventRecord(e1, s);
            net->ev_used.push_back({e0, e1, VF_KERNEL_DENSE_FWD_TC, 2.0 * (double)M * K * N});
        }
        return VF_OK;
    }
    if (absw)
        LAUNCH(net, launch_abs_rows_times_wt(A, nd.Wabs, (int)M, K, N, out, s));
    else
        LAUNCH(net, launch_rows_times_wt(A, nd.W, bias, (int)M, K, N, out, s));
    return VF_OK;
}

struct IbpState {
    std::vector<float*> c, r;
};

int run_ibp(vf_net* net, const float* centres, int B, float eps, Arena& ar, IbpState& st, cudaStream_t s,
            const signed char* const* split = nullptr, int sound = 0) {
    const size_t N = net->nodes.size();
    st.c.assign(N, nullptr);
    st.r.assign(N, nullptr);
    for (size_t v = 0; v < N; ++v) {
        const Node& nd = net->nodes[v];
        const long long cnt = (long long)B * nd.n;
        if (v == 0) {
            st.c[0] = const_cast<float*>(centres);
            st.r[0] = ar.take<float>(cnt);
            if (!st.r[0]) return fail(VF_ERR_WORKSPACE, "workspace too small for IBP buffers");
            LAUNCH(net, launch_fill(st.r[0], cnt, eps, s));
            continue;
        }
        st.c[v] = ar.take<float>(cnt);
        st.r[v] = ar.take<float>(cnt);
        if (!st.c[v] || !st.r[v]) return fail(VF_ERR_WORKSPACE, "workspace too small for IBP buffers");
        const int sv = nd.src;
        const long long cnt_src = (long long)B * net->nodes[sv].n;
        Arena tmp = ar;  // sound mode: |c| + r of the source and |W| (|c| + r), used at once
        float* T = sound ? tmp.take<float>(cnt_src) : nullptr;
        float* S = sound ? tmp.take<float>(cnt) : nullptr;
        if (sound && (!T || !S)) return fail(VF_ERR_WORKSPACE, "workspace too small for sound IBP");
        switch (nd.op) {
            case VF_DENSE:
                // IBP products stay on the FFMA kernel: on the tensor cores (3xTF32) the bounds of the
                // 3072-1024x8-100 network drifted from the fp64 oracle by up to 1.06x the parity tolerance after
                // eight layers (FFMA: 0.02x), and they are under 0.5% of any step
                if (!sound && net->fwd_tc == 3 && fwd_tc_ok(net, nd, st.c[sv], B, (int)net->nodes[sv].n) &&
                    (sv == 0 || fwd_tc_ok(net, nd, st.r[sv], B, (int)net->nodes[sv].n))) {
                    TRY(fwd_product(net, nd, st.c[sv], B, (int)net->nodes[sv].n, false, nd.b, st.c[v], s));
                    if (sv == 0)
                        LAUNCH(net, launch_ibp_radius_rowsum(nd.rowsum_abs, eps, B, (int)nd.n, st.r[v], s));
                    else
                        TRY(fwd_product(net, nd, st.r[sv], B, (int)net->nodes[sv].n, true, nullptr, st.r[v], s));
                    break;
                }
                LAUNCH(net, launch_ibp_dense(st.c[sv], st.r[sv], nd.W, nd.Wabs, nd.b, sv == 0 ? nd.rowsum_abs : nullptr,
                                             eps, B, (int)net->nodes[sv].n, (int)nd.n, st.c[v], st.r[v], s));
                if (sound) {  // every dot product of K terms errs by at most gamma_K (|W| (|c| + r) + |b|)
                    LAUNCH(net, launch_abs_plus(st.c[sv], st.r[sv], cnt_src, T, s));
                    LAUNCH(net, launch_abs_rows_times_wt(T, nd.Wabs, B, (int)net->nodes[sv].n, (int)nd.n, S, s));
                    LAUNCH(net, launch_sound_radius(st.r[v], S, nd.b, cnt, nd.n, 1, gamma_up(2 * net->nodes[sv].n + 64), s));
                }
                break;
            case VF_CONV2D: {
                const ConvGeom g = conv_geom(net, nd);
                LAUNCH(net, launch_ibp_conv(st.c[sv], st.r[sv], nd.W, nd.Wabs, nd.b, B, g, st.c[v], st.r[v], s));
                if (sound) {
                    LAUNCH(net, launch_abs_plus(st.c[sv], st.r[sv], cnt_src, T, s));
                    LAUNCH(net, launch_ibp_conv(T, nullptr, nd.Wabs, nd.Wabs, nullptr, B, g, S, nullptr, s));
                    LAUNCH(net, launch_sound_radius(st.r[v], S, nd.b, cnt, nd.n, (long long)g.ho * g.wo,
                                                    gamma_up(2LL * g.ci * g.k * g.k + 64), s));
                }
                break;
            }
            case VF_RELU:
                if (sound)
                    LAUNCH(net, launch_sound_relu(st.c[sv], st.r[sv], cnt, split ? split[v] : nullptr, st.c[v], st.r[v], s));
                else
                    LAUNCH(net, launch_ibp_relu(st.c[sv], st.r[sv], cnt, st.c[v], st.r[v], s, split ? split[v] : nullptr));
                break;
            case VF_ADD:
                if (sound)
                    LAUNCH(net, launch_sound_add(st.c[sv], st.r[sv], st.c[nd.src2], st.r[nd.src2], cnt, st.c[v], st.r[v], s));
                else
                    LAUNCH(net, launch_ibp_add(st.c[sv], st.r[sv], st.c[nd.src2], st.r[nd.src2], cnt, st.c[v], st.r[v], s));
                break;
        }
    }
    return VF_OK;
}

long long offset_of(const vf_net* net, int v, int B) {
    long long o = 0;
    for (int u = 0; u < v; ++u) o += net->nodes[u].n;
    return o * B;
}

// Enqueues the NaN/Inf scan of the arrays into a device flag; the flag is read back (with the
// compaction counts) by prepare_bounds, so a call synchronises its stream once.
int scan_finite_dev(vf_net* net, const std::vector<std::pair<const float*, long long>>& arrays, Arena& ar,
                    cudaStream_t s, int** flag_out) {
    int* flag = ar.take<int>(1);
    if (!flag) return fail(VF_ERR_WORKSPACE, "workspace too small");
    CU(cudaMemsetAsync(flag, 0, sizeof(int), s));
    for (auto& a : arrays)
        if (a.first != nullptr) LAUNCH(net, launch_finite_scan(a.first, a.second, flag, s));
    *flag_out = flag;
    return VF_OK;
}

// Runs every row block of one pass. `init` describes the start rows (global addressing).
int run_pass(vf_net* net, int start, Entry init, long long rows, long long R_pass, Arena& ar,
             const std::vector<const float4*>& relax, const float* centres, float eps, float* pass_out, float* ext_in,
             float* const_out, cudaStream_t s, const int* idx = nullptr, const std::vector<float*>* sw = nullptr) {
    const bool ext = ext_in != nullptr;
    const Node& sn = net->nodes[start];
    // rows held as receptive-field windows: identity-trick passes that start at a convolution or a residual
    // add (not in sound mode, whose rounding budget reads plain rows)
    const bool win_on = net->windows && !ext && sw == nullptr && init.kind == E_IDENT &&
                        (sn.op == VF_CONV2D || sn.op == VF_ADD) && sn.h > 1;
    int nb = 0;
    long long max_len = 0;
    TRY(pool_size(net, start, init, &relax, ext, win_on, idx != nullptr, &nb, &max_len, sw));
    long long nmax = (max_node_size(net, input_buffered(net) || sw != nullptr) + 31) / 32 * 32;  // 128-byte rows
    if (win_on) nmax = std::max<long long>(32, (max_len + 31) / 32 * 32);
    int tiles = std::max(dense_back_tiles_n((int)net->nodes[0].n), dense_back_tc_tiles_n((int)net->nodes[0].n));
    for (size_t v = 1; v < net->nodes.size(); ++v)  // per-tile partials of every convolution step
        if (net->nodes[v].op == VF_CONV2D) tiles = std::max(tiles, conv_back_tiles(conv_geom(net, net->nodes[v])));
    Arena a2 = ar;
    const size_t per_row = sizeof(float) * (1 + (size_t)tiles + (size_t)nb * nmax) + 64;
    long long chunk = (long long)(a2.left() / per_row);
    if (chunk > rows) chunk = rows;
    if (chunk >= 256) chunk -= chunk % 128;
    if (chunk < 1) return fail(VF_ERR_WORKSPACE, "workspace too small for one row of the pass");
    Walker w;
    w.net = net;
    w.s = s;
    w.dry = false;
    w.cst = a2.take<float>(chunk);
    w.part = a2.take<float>((size_t)chunk * tiles);
    w.ld_buf = nmax;
    w.bufs.assign(nb, nullptr);
    w.ref.assign(nb, 0);
    for (int i = 0; i < nb; ++i) w.bufs[i] = a2.take<float>((size_t)chunk * nmax);
    if (!w.cst || !w.part) return fail(VF_ERR_WORKSPACE, "workspace too small");
    for (int i = 0; i < nb; ++i)
        if (!w.bufs[i]) return fail(VF_ERR_WORKSPACE, "workspace too small");
    w.relax = &relax;
    w.centres = centres;
    w.eps = eps;
    w.n_centres = rows / R_pass;
    w.win_on = win_on;
    w.compact = idx != nullptr;
    w.sw = sw;
    w.ps = PassStart{sn.n, sn.h, sn.w};
    for (long long m0 = 0; m0 < rows; m0 += chunk) {
        w.M = std::min(chunk, rows - m0);
        w.pg = PassGeom{m0, R_pass, idx};
        Entry e = init;
        if (e.kind == E_VIRT) e.ref.m0 = m0;
        w.ext_in = ext ? ext_in + m0 * net->nodes[0].n : nullptr;
        TRY(w.run(start, e));
        if (pass_out != nullptr) LAUNCH(net, launch_finish_rows(w.cst, w.part, w.part_tiles, w.M, pass_out + m0, s));
        if (const_out != nullptr) CU(cudaMemcpyAsync(const_out + m0, w.cst, sizeof(float) * w.M,
                                                     cudaMemcpyDeviceToDevice, s));
    }
    return VF_OK;
}

int check_net(const vf_net* net) {
    if (net == nullptr) return fail(VF_ERR_ARG, "net is NULL");
    return VF_OK;
}

// Relaxation parameters for every ReLU from bounds arrays (vf_ibp layout) and optional alpha.
int build_relax(vf_net* net, int B, const std::vector<const float*>& L, const std::vector<const float*>& U,
                const float* const* alpha, Arena& ar, std::vector<const float4*>& relax, cudaStream_t s) {
    relax.assign(net->nodes.size(), nullptr);
    for (size_t v = 0; v < net->nodes.size(); ++v) {
        const Node& nd = net->nodes[v];
        if (nd.op != VF_RELU) continue;
        float4* P = ar.take<float4>((size_t)B * nd.n);
        if (!P) return fail(VF_ERR_WORKSPACE, "workspace too small for relaxation parameters");
        const Node& sn = net->nodes[nd.src];
        const bool aff = sn.op == VF_DENSE || sn.op == VF_CONV2D;
        LAUNCH(net, launch_relax_params(L[nd.src], U[nd.src], alpha ? alpha[v] : nullptr, (long long)B * nd.n, P,
                                        aff ? sn.b : nullptr, nd.n, sn.op == VF_CONV2D ? (long long)sn.h * sn.w : 1, s));
        relax[v] = P;
    }
    return VF_OK;
}

// Bounds of every ReLU source (IBP, refined by CROWN passes where asked) and the relaxation tables.
struct Bounds {
    std::vector<float*> Lw, Uw;
    std::vector<const float4*> relax;
    // sound mode: sw[v] [B, n_v], the rounding weights of node v (per unit of a row's coefficient magnitude
    // over v's output; computed for nodes [0, a_next))
    std::vector<float*> sw;
    int a_next = 0;
};

// Magnitude bound M_v >= |value of node v| over the box (sound bounds): from refined bounds where a node
// feeds a ReLU, max(u, 0) of the source for a ReLU output, |c| + r from interval propagation otherwise.
int magnitude_of(vf_net* net, int v, int B, const IbpState& st, const Bounds& bd, float* M, cudaStream_t s) {
    const Node& nd = net->nodes[v];
    const long long cnt = (long long)B * nd.n;
    if (nd.op == VF_RELU && bd.Lw[nd.src] != nullptr) {
        LAUNCH(net, launch_magnitude(bd.Lw[nd.src], bd.Uw[nd.src], cnt, 1, M, s));
    } else if (bd.Lw[v] != nullptr) {
        LAUNCH(net, launch_magnitude(bd.Lw[v], bd.Uw[v], cnt, 0, M, s));
    } else {
        LAUNCH(net, launch_abs_plus(st.c[v], st.r[v], cnt, M, s));
    }
    return VF_OK;
}

// Rounding weights w_v of nodes [bd.a_next, upto] (k_sound.cu states the analysis) into the arrays bd.sw
// (allocated by the caller); `scratch` holds transient vectors. A ReLU's weight needs its final bounds and
// relaxation; other nodes' weights may use bounds refined later (earlier bounds are valid, only wider).
int sound_weights(vf_net* net, int B, float eps, const float* centres, const IbpState& st, Bounds& bd, int upto,
                  Arena scratch, cudaStream_t s) {
    const float gN = gamma_up(net->total + 64);  // a row constant sums at most one term per neuron of the net
    for (int v = bd.a_next; v <= upto; ++v) {
        const Node& nd = net->nodes[v];
        const long long cnt = (long long)B * nd.n;
        float* w = bd.sw[v];
        Arena tmp = scratch;
        switch (nd.op) {
            case VF_INPUT:
                LAUNCH(net, launch_input_weight(centres, eps, cnt, gamma_up(2 * nd.n + 64), w, s));
                break;
            case VF_DENSE:
            case VF_CONV2D: {
                const Node& sn = net->nodes[nd.src];
                const long long cs = (long long)B * sn.n;
                float* Ms = tmp.take<float>(cs);
                float* Mv = tmp.take<float>(cnt);
                if (!Ms || !Mv) return fail(VF_ERR_WORKSPACE, "workspace too small for rounding weights");
                TRY(magnitude_of(net, nd.src, B, st, bd, Ms, s));
                TRY(magnitude_of(net, v, B, st, bd, Mv, s));
                long long kb, kf, per_channel = 1;  // terms of one backward / forward dot product
                ConvGeom g{};
                if (nd.op == VF_DENSE) {
                    kb = nd.n;
                    kf = sn.n;
                    LAUNCH(net, launch_abs_rows_times_wt(Ms, nd.Wabs, B, (int)sn.n, (int)nd.n, w, s));
                } else {
                    g = conv_geom(net, nd);
                    kb = (long long)g.co * g.k * g.k;
                    kf = (long long)g.ci * g.k * g.k;
                    per_channel = (long long)g.ho * g.wo;
                    LAUNCH(net, launch_ibp_conv(Ms, nullptr, nd.Wabs, nd.Wabs, nullptr, B, g, w, nullptr, s));
                }
                const float gb = gamma_up(kb + 64);
                const float gQ = nextafterf(gb * (1.f + 2.f * gamma_up(kf + 64)), INFINITY);
                LAUNCH(net, launch_affine_weight(w, nd.b, Mv, cnt, nd.n, per_channel, gQ, gN, s));
                break;
            }
            case VF_RELU:
                LAUNCH(net, launch_relu_weight(bd.relax[v], bd.Lw[nd.src], bd.Uw[nd.src], cnt, gN, w, s));
                break;
            default: {  // add: the rows' sums at its sources are charged there
                float* Mv = tmp.take<float>(cnt);
                if (!Mv) return fail(VF_ERR_WORKSPACE, "workspace too small for rounding weights");
                TRY(magnitude_of(net, v, B, st, bd, Mv, s));
                LAUNCH(net, launch_scale_up(Mv, cnt, 0x1p-23f, w, s));
                break;
            }
        }
    }
    bd.a_next = std::max(bd.a_next, upto + 1);
    return VF_OK;
}

bool affine_chain(const vf_net* net);
int alpha_chain(vf_net* net, int L, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                const vf_opts& o, int iters, float lr, bool grad_mode, const float* alpha_in, float* grad_out,
                float* lb, float* lb_start, float* alpha_out, const Bounds& bd, Arena ar, cudaStream_t s,
                const float* beta_in, float* beta_grad_out, const int* unit_idx = nullptr);

int prepare_bounds(vf_net* net, const float* centres, int B, float eps, const vf_opts& o, Arena& ar, IbpState& st,
                   Bounds& bd, cudaStream_t s, const int* finite_flag = nullptr) {
    const int nn = (int)net->nodes.size();
    const int sound = o.sound ? 1 : 0;
    TRY(run_ibp(net, centres, B, eps, ar, st, s, o.split, sound));
    bd.Lw.assign(nn, nullptr);
    bd.Uw.assign(nn, nullptr);
    bd.relax.assign(nn, nullptr);
    std::vector<float4*> P(nn, nullptr);
    long long max_pass_rows = 1;
    for (int v = 0; v < nn; ++v)
        if (net->nodes[v].op == VF_RELU) {
            P[v] = ar.take<float4>((size_t)B * net->nodes[v].n);
            if (!P[v]) return fail(VF_ERR_WORKSPACE, "workspace too small for relaxation parameters");
            bd.relax[v] = P[v];
            max_pass_rows = std::max(max_pass_rows, 2 * net->nodes[v].n);
        }
    // A ReLU whose bounds no CROWN pass refines (IBP substitution, or an exact source) takes its
    // relaxation in the same pass that forms its bounds from the IBP centre and radius.
    auto refined = [&](int k) {
        const bool crown = (o.relu_crown == nullptr) || (o.relu_crown[k] != 0);
        return crown && !exact_source(net, net->nodes[k].src);
    };
    auto relax_args = [&](int k, const float** bias, long long* per_channel) {
        const Node& sn = net->nodes[net->nodes[k].src];
        const bool aff = sn.op == VF_DENSE || sn.op == VF_CONV2D;
        *bias = aff ? sn.b : nullptr;
        *per_channel = sn.op == VF_CONV2D ? (long long)sn.h * sn.w : 1;
    };
    for (int v = 0; v < nn; ++v) {
        if (net->nodes[v].op != VF_RELU) continue;
        const int p = net->nodes[v].src;
        const long long cnt = (long long)B * net->nodes[p].n;
        bd.Lw[p] = ar.take<float>(cnt);
        bd.Uw[p] = ar.take<float>(cnt);
        if (!bd.Lw[p] || !bd.Uw[p]) return fail(VF_ERR_WORKSPACE, "workspace too small for intermediate bounds");
        if (!refined(v)) {
            const float* bias;
            long long pc;
            relax_args(v, &bias, &pc);
            LAUNCH(net, launch_relu_bounds_relax(st.c[p], st.r[p], o.split ? o.split[v] : nullptr, nullptr, bd.Lw[p],
                                                 bd.Uw[p], o.alpha ? o.alpha[v] : nullptr, B, net->nodes[p].n, P[v],
                                                 bias, pc, sound, s));
        } else {
            LAUNCH(net, launch_bounds_from_cr(st.c[p], st.r[p], cnt, bd.Lw[p], bd.Uw[p], s,
                                              o.split ? o.split[v] : nullptr, sound));
        }
    }
    if (sound) {  // error weights of every node, kept for the specification pass
        bd.sw.assign(nn, nullptr);
        bd.a_next = 0;
        for (int v = 0; v < nn; ++v) {
            bd.sw[v] = ar.take<float>((size_t)B * net->nodes[v].n);
            if (!bd.sw[v]) return fail(VF_ERR_WORKSPACE, "workspace too small for error weights");
        }
    }
    // Unstable-neuron compaction: only IBP-unstable neurons change at the intersection, so a pass needs
    // rows for those alone. The number per centre is read back once (one host synchronisation) and each
    // pass is sized for the largest count; a pass whose largest count is above 7/8 of the node stays plain.
    // The finite-check flag (if any) is read back in the same copy, before any pass runs.
    std::vector<int> half(nn, -1);  // -1: plain pass, 0: nothing to refine, > 0: compacted rows per sign
    std::vector<int> ps;
    if (net->compact && !o.no_host_sync)
        for (int k = 0; k < nn; ++k) {
            const int p = net->nodes[k].src;
            if (net->nodes[k].op == VF_RELU && ((o.relu_crown == nullptr) || (o.relu_crown[k] != 0)) &&
                !exact_source(net, p))
                ps.push_back(p);
        }
    if (!ps.empty() || finite_flag != nullptr) {
        int* counts = ar.take<int>(1 + (size_t)B * ps.size());  // [0]: finite flag, then [pass][centre]
        if (!counts) return fail(VF_ERR_WORKSPACE, "workspace too small");
        if (finite_flag != nullptr)
            CU(cudaMemcpyAsync(counts, finite_flag, sizeof(int), cudaMemcpyDeviceToDevice, s));
        else
            CU(cudaMemsetAsync(counts, 0, sizeof(int), s));
        for (size_t i = 0; i < ps.size(); ++i)
            LAUNCH(net, launch_unstable_count(bd.Lw[ps[i]], bd.Uw[ps[i]], B, net->nodes[ps[i]].n, counts + 1 + i * B, s));
        std::vector<int> h(1 + (size_t)B * ps.size());
        CU(cudaMemcpyAsync(h.data(), counts, sizeof(int) * h.size(), cudaMemcpyDeviceToHost, s));
        CU(cudaStreamSynchronize(s));
        if (h[0]) return fail(VF_ERR_NONFINITE, "NaN or Inf in centres, C or alpha");
        for (size_t i = 0; i < ps.size(); ++i) {
            const int u_max = *std::max_element(h.begin() + 1 + i * B, h.begin() + 1 + (i + 1) * B);
            half[ps[i]] = (8LL * u_max <= 7LL * net->nodes[ps[i]].n) ? u_max : -1;
        }
    }
    Arena tmp = ar;  // pass outputs are transient
    float* pass_out = tmp.take<float>((size_t)B * max_pass_rows);
    if (!pass_out) return fail(VF_ERR_WORKSPACE, "workspace too small");
    // alpha-CROWN for the bounds of ReLU k's dense source p, right after its CROWN pass: the neurons still
    // unstable take rows [e_j; -e_j] over p, ascended (per-row slopes of the earlier ReLUs, split multipliers
    // where splits are given) on the network up to p; their bounds become max / min with the best iterate, and
    // the relaxation of k is formed again.
    const bool chain = affine_chain(net);
    auto inter_alpha = [&](int k) -> int {
        const int p = net->nodes[k].src;
        if (o.alpha_inter_iters <= 0 || sound || !refined(k) || net->nodes[p].op != VF_DENSE) return VF_OK;
        if (!chain) return fail(VF_ERR_UNSUPPORTED, "intermediate alpha optimisation covers chain networks");
        const long long np = net->nodes[p].n;
        Arena t2 = tmp;
        int* cnt = t2.take<int>(B);
        if (!cnt) return fail(VF_ERR_WORKSPACE, "workspace too small");
        LAUNCH(net, launch_unstable_count(bd.Lw[p], bd.Uw[p], B, np, cnt, s));
        std::vector<int> h(B);
        CU(cudaMemcpyAsync(h.data(), cnt, sizeof(int) * B, cudaMemcpyDeviceToHost, s));
        CU(cudaStreamSynchronize(s));
        const int hp = *std::max_element(h.begin(), h.end());
        if (hp == 0) return VF_OK;
        int* idx = t2.take<int>((size_t)B * hp);
        float* best = t2.take<float>((size_t)B * 2 * hp);
        if (!idx || !best) return fail(VF_ERR_WORKSPACE, "workspace too small for intermediate alpha rows");
        LAUNCH(net, launch_unstable_list(bd.Lw[p], bd.Uw[p], B, np, hp, idx, s));
        vf_opts oi = o;  // the start states and outputs of a specification ascent do not apply here
        oi.alpha_rows_init = nullptr;
        oi.beta_rows_init = nullptr;
        oi.beta_rows_out = nullptr;
        TRY(alpha_chain(net, p, centres, B, eps, nullptr, 2 * hp, 0, oi, o.alpha_inter_iters, o.alpha_inter_lr, false,
                        nullptr, nullptr, best, nullptr, nullptr, bd, t2, s, nullptr, nullptr, idx));
        LAUNCH(net, launch_intersect_compact(bd.Lw[p], bd.Uw[p], best, idx, B, np, hp, s));
        const float* bias;
        long long pc;
        relax_args(k, &bias, &pc);
        LAUNCH(net, launch_relax_params(bd.Lw[p], bd.Uw[p], o.alpha ? o.alpha[k] : nullptr, (long long)B * net->nodes[k].n,
                                        P[k], bias, net->nodes[k].n, pc, s, sound));
        return VF_OK;
    };
    for (int k = 0; k < nn; ++k) {
        const Node& nd = net->nodes[k];
        if (nd.op != VF_RELU) continue;
        const int p = nd.src;
        const bool crown = (o.relu_crown == nullptr) || (o.relu_crown[k] != 0);
        const bool run = crown && !exact_source(net, p) && half[p] != 0;
        if (sound && run) TRY(sound_weights(net, B, eps, centres, st, bd, p, tmp, s));
        const std::vector<float*>* sw = sound ? &bd.sw : nullptr;
        if (crown && !exact_source(net, p) && half[p] > 0) {
            const long long np = net->nodes[p].n;
            const int hp = half[p];
            int* idx = tmp.take<int>((size_t)B * hp);
            if (!idx) return fail(VF_ERR_WORKSPACE, "workspace too small");
            LAUNCH(net, launch_unstable_list(bd.Lw[p], bd.Uw[p], B, np, hp, idx, s));
            Entry init;
            init.kind = E_IDENT;
            TRY(run_pass(net, p, init, (long long)B * 2 * hp, 2 * hp, tmp, bd.relax, centres, eps, pass_out, nullptr,
                         nullptr, s, idx, sw));
            LAUNCH(net, launch_intersect_compact(bd.Lw[p], bd.Uw[p], pass_out, idx, B, np, hp, s));
        } else if (crown && !exact_source(net, p) && half[p] < 0) {
            Entry init;
            init.kind = E_IDENT;
            const long long np = net->nodes[p].n;
            TRY(run_pass(net, p, init, (long long)B * 2 * np, 2 * np, tmp, bd.relax, centres, eps, pass_out, nullptr,
                         nullptr, s, nullptr, sw));
            // the intersection and the relaxation in one pass over the layer
            const float* bias;
            long long pc;
            relax_args(k, &bias, &pc);
            LAUNCH(net, launch_relu_bounds_relax(nullptr, nullptr, nullptr, pass_out, bd.Lw[p], bd.Uw[p],
                                                 o.alpha ? o.alpha[k] : nullptr, B, np, P[k], bias, pc, sound, s));
            TRY(inter_alpha(k));
            continue;
        }
        if (!refined(k)) continue;  // relaxed together with its bounds above
        const Node& sn = net->nodes[p];
        const bool aff = sn.op == VF_DENSE || sn.op == VF_CONV2D;
        LAUNCH(net, launch_relax_params(bd.Lw[p], bd.Uw[p], o.alpha ? o.alpha[k] : nullptr, (long long)B * nd.n, P[k],
                                        aff ? sn.b : nullptr, nd.n, sn.op == VF_CONV2D ? (long long)sn.h * sn.w : 1, s,
                                        sound));
        TRY(inter_alpha(k));
    }
    return VF_OK;
}

// A ReLU chain laid out input -> affine -> relu -> affine -> ... -> dense (nodes in that order), each
// affine node dense or a convolution.
bool affine_chain(const vf_net* net) {
    const int nn = (int)net->nodes.size();
    for (int v = 1; v < nn; ++v) {
        const Node& nd = net->nodes[v];
        if (nd.src != v - 1) return false;
        if (v % 2 == 1 ? (nd.op != VF_DENSE && nd.op != VF_CONV2D) : nd.op != VF_RELU) return false;
    }
    return net->nodes[nn - 1].op == VF_DENSE;
}

// alpha-CROWN on the specification rows of a dense chain: per-row lower slopes of unstable neurons.
// grad_mode: one evaluation at alpha_in, writing lb and d lb / d alpha (grad_out) -- no update.
// Otherwise: iters Adam ascent steps from the adaptive slopes, lb = best bound seen per row,
// lb_start (optional) = the bound at the adaptive start, alpha_out (optional) = the final slopes.
// Slope arrays: for each ReLU node in order, a [B, R, n] block.
// alpha-CROWN on a chain network (affine_chain) up to its node L, which is dense: rows C [B or 1, R, n_L] over
// node L's output, per-row slopes of every ReLU before L (and split multipliers where o.split is set), the
// relaxations of bd, scratch from ar. The specification pass (L = last node) and the intermediate passes of
// prepare_bounds (L = a ReLU's dense source) both run here. unit_idx (or null): the rows are [e_j; -e_j] per
// centre for the neurons listed as in a compacted identity-trick pass (R = 2 x entries per centre; C unused).
int alpha_chain(vf_net* net, int L, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                const vf_opts& o, int iters, float lr, bool grad_mode, const float* alpha_in, float* grad_out,
                float* lb, float* lb_start, float* alpha_out, const Bounds& bd, Arena ar, cudaStream_t s,
                const float* beta_in, float* beta_grad_out, const int* unit_idx) {
    const int nn = (int)net->nodes.size();
    const long long n0 = net->nodes[0].n;
    const int nL = (int)net->nodes[L].n;
    if (net->nodes[L].op != VF_DENSE) return fail(VF_ERR_UNSUPPORTED, "alpha optimisation needs rows over a dense node");
    std::vector<int> relus;
    long long sum_n = 0, nmax = 1;
    std::vector<long long> aoff(nn, 0);  // offset of each ReLU's [B, R, n] slope block
    for (int v = 2; v < L; v += 2) {
        relus.push_back(v);
        aoff[v] = (long long)B * R * sum_n;
        sum_n += net->nodes[v].n;
        nmax = std::max(nmax, net->nodes[v].n);
    }
    const long long gmax = std::max<long long>(nmax, n0);
    const long long rows = (long long)B * R;
    // identity relaxation table [B, nmax]: the slopes are applied by relax_alpha_rows_k, so the contraction
    // that follows may run on the tensor cores, which read every row through such a table
    float4* ident = nullptr;
    if (net->dense_kernel != 1 && !net->call_sound) {
        ident = ar.take<float4>((size_t)B * nmax);
        if (!ident) return fail(VF_ERR_WORKSPACE, "workspace too small for alpha optimisation");
        LAUNCH(net, launch_identity_relax(ident, (long long)B * nmax, s));
    }
    // per-row floats: H (sum_n) + Z (nmax) + lam_in (n0) + two gradient buffers (gmax) + cst + lb
    // (+ slopes and two Adam moments, 3 * sum_n, when optimising)
    int ctiles_max = 0;
    for (int v = 1; v < L; v += 2)
        if (net->nodes[v].op == VF_CONV2D) ctiles_max = std::max(ctiles_max, conv_back_tiles(conv_geom(net, net->nodes[v])));
    long long sum_split = 0;  // neurons of ReLUs with split constraints (their beta rows)
    for (int u : relus)
        if (o.split && o.split[u]) sum_split += net->nodes[u].n;
    const size_t per_row =
        sizeof(float) * (sum_n + nmax + n0 + 2 * gmax + 2 + ctiles_max + (grad_mode ? 0 : 3 * (sum_n + sum_split))) +
        64 * (2 * relus.size() + 8);
    long long chunk = (long long)(ar.left() / per_row);
    if (chunk > rows) chunk = rows;
    if (chunk < 1) return fail(VF_ERR_WORKSPACE, "workspace too small for alpha optimisation");
    std::vector<float*> H(nn, nullptr), A(nn, nullptr), M1(nn, nullptr), M2(nn, nullptr);
    std::vector<float*> Bt(nn, nullptr), BM1(nn, nullptr), BM2(nn, nullptr);
    for (int u : relus) {
        H[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
        if (!grad_mode) {
            A[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            M1[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            M2[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            if (o.split && o.split[u]) {
                Bt[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                BM1[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                BM2[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                if (!Bt[u] || !BM1[u] || !BM2[u]) return fail(VF_ERR_WORKSPACE, "workspace too small");
            }
        }
    }
    float* Z = ar.take<float>((size_t)chunk * nmax);
    float* lam_in = ar.take<float>((size_t)chunk * n0);
    float* G0 = ar.take<float>((size_t)chunk * gmax);
    float* G1 = ar.take<float>((size_t)chunk * gmax);
    float* cst = ar.take<float>(chunk);
    float* lbc = ar.take<float>(chunk);
    int ctiles = 0;  // per-tile partials written by the convolution kernel (unused here: no bias, no relaxation)
    for (int v = 1; v < L; v += 2)
        if (net->nodes[v].op == VF_CONV2D) ctiles = std::max(ctiles, conv_back_tiles(conv_geom(net, net->nodes[v])));
    float* cpart = ctiles ? ar.take<float>((size_t)chunk * ctiles) : nullptr;
    if (!Z || !lam_in || !G0 || !G1 || !cst || !lbc || (ctiles && !cpart))
        return fail(VF_ERR_WORKSPACE, "workspace too small");
    for (int u : relus)
        if (!H[u] || (!grad_mode && (!A[u] || !M1[u] || !M2[u]))) return fail(VF_ERR_WORKSPACE, "workspace too small");

    for (long long m0 = 0; m0 < rows; m0 += chunk) {
        const long long Mc = std::min(chunk, rows - m0);
        const PassGeom pg{m0, R};
        std::vector<float*> al(nn, nullptr);
        for (int u : relus) {
            const long long nu = net->nodes[u].n;
            if (grad_mode) {
                al[u] = const_cast<float*>(alpha_in) + aoff[u] + m0 * nu;
            } else {
                al[u] = A[u];
                const float* ai = o.alpha_rows_init ? o.alpha_rows_init + aoff[u] + m0 * nu : nullptr;
                LAUNCH(net, launch_alpha_init(A[u], M1[u], M2[u], Mc, (int)nu, bd.relax[u], pg, s, ai));
            }
        }
        std::vector<BetaRows> bt(nn);
        for (int u : relus) {
            if (!(o.split && o.split[u])) continue;
            const long long nu = net->nodes[u].n;
            bt[u].split = o.split[u];
            if (grad_mode) {
                bt[u].beta = beta_in ? const_cast<float*>(beta_in) + aoff[u] + m0 * nu : nullptr;
                bt[u].grad_out = beta_grad_out ? beta_grad_out + aoff[u] + m0 * nu : nullptr;
            } else {
                bt[u].beta = Bt[u];
                bt[u].m1 = BM1[u];
                bt[u].m2 = BM2[u];
                const float* bi = o.beta_rows_init ? o.beta_rows_init + aoff[u] + m0 * nu : nullptr;
                LAUNCH(net, launch_zero_moments(Bt[u], BM1[u], BM2[u], Mc * nu, s, bi));
            }
        }
        const int evals = grad_mode ? 1 : iters + 1;
        for (int it = 0; it < evals; ++it) {
            // down: back-substitution of the rows with the current slopes, keeping lam over every ReLU
            CU(cudaMemsetAsync(cst, 0, sizeof(float) * Mc, s));
            const Node& last = net->nodes[L];
            if (unit_idx != nullptr) {  // rows [e_j; -e_j]: the first step gathers +-W[j, :] and adds +-b[j]
                const PassGeom pgi{m0, R, unit_idx};
                LAUNCH(net, launch_gather_start_rows(H[L - 1], net->nodes[L - 1].n, Mc, pgi, last.W, nL,
                                                     net->nodes[L - 1].n, s));
                LAUNCH(net, launch_cst_identity_bias(cst, Mc, pgi, last.b, nL, 1, s));
            } else {
                LAUNCH(net, launch_dense_back(RowRef{C, C_bstride, nL, R, m0}, Relax{nullptr, 0}, last.W, last.b, Mc,
                                              nL, (int)net->nodes[L - 1].n, pg, OUT_STORE, H[L - 1],
                                              net->nodes[L - 1].n, cst, nullptr, 0.f, nullptr, s));
            }
            for (int u = L - 1; u >= 2; u -= 2) {
                const int nu = (int)net->nodes[u].n;
                const Node& d = net->nodes[u - 1];
                const int nd_in = (int)net->nodes[u - 2].n;
                LAUNCH(net, launch_relax_alpha_rows(H[u], Mc, nu, bd.relax[u], pg, al[u], Z, cst, s, 1, 0, bt[u]));
                float* out = (u - 2 == 0) ? lam_in : H[u - 2];
                if (d.op == VF_CONV2D)
                    LAUNCH(net, launch_conv_back(RowRef{Z, 0, nu, kHugeRows, 0}, Relax{nullptr, 0}, d.W, nullptr, Mc,
                                                 conv_geom(net, d), pg, OUT_STORE, out, nd_in, cpart, nullptr, 0.f,
                                                 net->num_sms, s));
                else if (ident != nullptr && d.WtHi != nullptr && back_tc_ok(net, Mc, nd_in) &&
                         dense_back_tc_supported(RowRef{Z, 0, nu, kHugeRows, 0}, Relax{ident, 0}, Mc, nu, nd_in, pg))
                    LAUNCH(net, launch_dense_back_tc(RowRef{Z, 0, nu, kHugeRows, 0}, Relax{ident, 0}, d.WtHi, d.WtLo, B,
                                                     Mc, nu, nd_in, pg, OUT_STORE, out, nd_in, cst, nullptr, 0.f,
                                                     nullptr, net->d_err, 0, s));
                else
                    LAUNCH(net, launch_dense_back(RowRef{Z, 0, nu, kHugeRows, 0}, Relax{nullptr, 0}, d.W, nullptr, Mc,
                                                  nu, nd_in, pg, OUT_STORE, out, nd_in, nullptr, nullptr, 0.f, nullptr,
                                                  s));
            }
            LAUNCH(net, launch_concretize_grad(lam_in, Mc, (int)n0, pg, centres, eps, cst, lbc, G0, s));
            if (it == 0 && lb_start) CU(cudaMemcpyAsync(lb_start + m0, lbc, sizeof(float) * Mc, cudaMemcpyDeviceToDevice, s));
            LAUNCH(net, launch_best_update(lb + m0, lbc, Mc, it == 0 ? 1 : 0, s));
            if (!grad_mode && it == iters) break;
            // up: gradient with respect to every ReLU's slopes (and one Adam ascent step)
            float* G = G0;
            float* Gn = G1;
            for (int d = 1; d + 1 < L; d += 2) {
                const Node& dn = net->nodes[d];
                const int u = d + 1;
                const int nu = (int)net->nodes[u].n;
                if (dn.op == VF_CONV2D)
                    LAUNCH(net, launch_ibp_conv(G, nullptr, dn.W, dn.Wabs, dn.b, (int)Mc, conv_geom(net, dn), Gn,
                                                nullptr, s));
                else
                    TRY(fwd_product(net, dn, G, Mc, (int)net->nodes[d - 1].n, false, dn.b, Gn, s));
                float* gout = grad_mode ? grad_out + aoff[u] + m0 * nu : nullptr;
                LAUNCH(net, launch_relax_grad_adam(Gn, H[u], Mc, nu, bd.relax[u], pg, al[u], gout, M1[u], M2[u],
                                                   grad_mode ? 0 : it + 1, lr, s, bt[u]));
                std::swap(G, Gn);
            }
        }
        if (!grad_mode && alpha_out)
            for (int u : relus) {
                const long long nu = net->nodes[u].n;
                CU(cudaMemcpyAsync(alpha_out + aoff[u] + m0 * nu, A[u], sizeof(float) * Mc * nu,
                                   cudaMemcpyDeviceToDevice, s));
            }
        if (!grad_mode && o.beta_rows_out)
            for (int u : relus) {
                const long long nu = net->nodes[u].n;
                if (Bt[u] != nullptr)
                    CU(cudaMemcpyAsync(o.beta_rows_out + aoff[u] + m0 * nu, Bt[u], sizeof(float) * Mc * nu,
                                       cudaMemcpyDeviceToDevice, s));
                else
                    CU(cudaMemsetAsync(o.beta_rows_out + aoff[u] + m0 * nu, 0, sizeof(float) * Mc * nu, s));
            }
    }
    return VF_OK;
}

int spec_alpha(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
               const vf_opts& o, int iters, float lr, bool grad_mode, const float* alpha_in, float* grad_out,
               float* lb, float* lb_start, float* alpha_out, cudaStream_t s, const float* beta_in = nullptr,
               float* beta_grad_out = nullptr) {
    Arena ar{net->ws, net->ws_bytes};
    IbpState st;
    Bounds bd;
    TRY(prepare_bounds(net, centres, B, eps, o, ar, st, bd, s));
    return alpha_chain(net, (int)net->nodes.size() - 1, centres, B, eps, C, R, C_bstride, o, iters, lr, grad_mode,
                       alpha_in, grad_out, lb, lb_start, alpha_out, bd, ar, s, beta_in, beta_grad_out);
}

// alpha-CROWN on any node graph (residual adds included): the same computation as spec_alpha with every
// node's coefficients materialised. Down: pending rows per node (the first contribution stores, later
// ones add), affine nodes add their bias to the row constant, ReLUs apply per-row slopes and keep the
// rows over their output for the gradient. Up, in topological order: G over each node's output from its
// sources' G (affine: forward product plus bias; ReLU: the slope chain rule and the slope gradient /
// Adam step; add: sum of the two sources).
int spec_alpha_graph(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                     const vf_opts& o, int iters, float lr, bool grad_mode, const float* alpha_in, float* grad_out,
                     float* lb, float* lb_start, float* alpha_out, cudaStream_t s, const float* beta_in = nullptr,
                     float* beta_grad_out = nullptr) {
    const int nn = (int)net->nodes.size();
    const int L = nn - 1;
    const long long n0 = net->nodes[0].n;
    const int nL = (int)net->nodes[L].n;
    if (net->nodes[L].op != VF_DENSE) return fail(VF_ERR_UNSUPPORTED, "alpha optimisation needs a dense last node");
    Arena ar{net->ws, net->ws_bytes};
    IbpState st;
    Bounds bd;
    TRY(prepare_bounds(net, centres, B, eps, o, ar, st, bd, s));
    std::vector<int> relus;
    long long sum_relu = 0, sum_all = 0;
    std::vector<long long> aoff(nn, 0);
    int ctiles = 0;
    for (int v = 0; v < nn; ++v) {
        const Node& nd = net->nodes[v];
        sum_all += nd.n;
        if (nd.op == VF_RELU) {
            relus.push_back(v);
            aoff[v] = (long long)B * R * sum_relu;
            sum_relu += nd.n;
        }
        if (nd.op == VF_CONV2D) ctiles = std::max(ctiles, conv_back_tiles(conv_geom(net, nd)));
    }
    const long long rows = (long long)B * R;
    long long sum_split = 0;  // neurons of ReLUs with split constraints (their beta rows)
    for (int u : relus)
        if (o.split && o.split[u]) sum_split += net->nodes[u].n;
    // per row: pending rows and gradients of every node, the per-ReLU slopes and Adam moments (and the
    // multipliers of split ReLUs with theirs), constants
    const size_t per_row = sizeof(float) * (2 * sum_all + (grad_mode ? 0 : 3 * (sum_relu + sum_split)) + 2 + ctiles) +
                           64 * (2 * nn + 6 * relus.size() + 8);
    long long chunk = (long long)(ar.left() / per_row);
    if (chunk > rows) chunk = rows;
    if (chunk < 1) return fail(VF_ERR_WORKSPACE, "workspace too small for alpha optimisation");
    std::vector<float*> P(nn, nullptr), G(nn, nullptr), A(nn, nullptr), M1(nn, nullptr), M2(nn, nullptr);
    for (int v = 0; v < nn; ++v) {
        P[v] = ar.take<float>((size_t)chunk * net->nodes[v].n);
        G[v] = ar.take<float>((size_t)chunk * net->nodes[v].n);
        if (!P[v] || !G[v]) return fail(VF_ERR_WORKSPACE, "workspace too small");
    }
    std::vector<float*> Bt(nn, nullptr), BM1(nn, nullptr), BM2(nn, nullptr);
    for (int u : relus)
        if (!grad_mode) {
            A[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            M1[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            M2[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
            if (!A[u] || !M1[u] || !M2[u]) return fail(VF_ERR_WORKSPACE, "workspace too small");
            if (o.split && o.split[u]) {
                Bt[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                BM1[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                BM2[u] = ar.take<float>((size_t)chunk * net->nodes[u].n);
                if (!Bt[u] || !BM1[u] || !BM2[u]) return fail(VF_ERR_WORKSPACE, "workspace too small");
            }
        }
    float* cst = ar.take<float>(chunk);
    float* lbc = ar.take<float>(chunk);
    float* cpart = ctiles ? ar.take<float>((size_t)chunk * ctiles) : nullptr;
    if (!cst || !lbc || (ctiles && !cpart)) return fail(VF_ERR_WORKSPACE, "workspace too small");

    for (long long m0 = 0; m0 < rows; m0 += chunk) {
        const long long Mc = std::min(chunk, rows - m0);
        const PassGeom pg{m0, R};
        std::vector<float*> al(nn, nullptr);
        for (int u : relus) {
            const long long nu = net->nodes[u].n;
            if (grad_mode) {
                al[u] = const_cast<float*>(alpha_in) + aoff[u] + m0 * nu;
            } else {
                al[u] = A[u];
                const float* ai = o.alpha_rows_init ? o.alpha_rows_init + aoff[u] + m0 * nu : nullptr;
                LAUNCH(net, launch_alpha_init(A[u], M1[u], M2[u], Mc, (int)nu, bd.relax[u], pg, s, ai));
            }
        }
        std::vector<BetaRows> bt(nn);
        for (int u : relus) {
            if (!(o.split && o.split[u])) continue;
            const long long nu = net->nodes[u].n;
            bt[u].split = o.split[u];
            if (grad_mode) {
                bt[u].beta = beta_in ? const_cast<float*>(beta_in) + aoff[u] + m0 * nu : nullptr;
                bt[u].grad_out = beta_grad_out ? beta_grad_out + aoff[u] + m0 * nu : nullptr;
            } else {
                bt[u].beta = Bt[u];
                bt[u].m1 = BM1[u];
                bt[u].m2 = BM2[u];
                const float* bi = o.beta_rows_init ? o.beta_rows_init + aoff[u] + m0 * nu : nullptr;
                LAUNCH(net, launch_zero_moments(Bt[u], BM1[u], BM2[u], Mc * nu, s, bi));
            }
        }
        const int evals = grad_mode ? 1 : iters + 1;
        for (int it = 0; it < evals; ++it) {
            // ---- down: pending rows per node; written[v]: P[v] holds a first contribution
            std::vector<char> written(nn, 0);
            CU(cudaMemsetAsync(cst, 0, sizeof(float) * Mc, s));
            const Node& last = net->nodes[L];
            LAUNCH(net, launch_dense_back(RowRef{C, C_bstride, nL, R, m0}, Relax{nullptr, 0}, last.W, last.b, Mc, nL,
                                          (int)net->nodes[last.src].n, pg, OUT_STORE, P[last.src],
                                          net->nodes[last.src].n, cst, nullptr, 0.f, nullptr, s));
            written[last.src] = 1;
            for (int v = L - 1; v >= 1; --v) {
                if (!written[v]) continue;
                const Node& nd = net->nodes[v];
                const int nv = (int)nd.n;
                const RowRef rv{P[v], 0, nv, kHugeRows, 0};
                auto mode_of = [&](int src) { return written[src] ? OUT_ACCUM : OUT_STORE; };
                switch (nd.op) {
                    case VF_DENSE: {
                        const int ns = (int)net->nodes[nd.src].n;
                        LAUNCH(net, launch_dense_back(rv, Relax{nullptr, 0}, nd.W, nd.b, Mc, nv, ns, pg, mode_of(nd.src),
                                                      P[nd.src], ns, cst, nullptr, 0.f, nullptr, s));
                        written[nd.src] = 1;
                        break;
                    }
                    case VF_CONV2D: {
                        const ConvGeom g = conv_geom(net, nd);
                        LAUNCH(net, launch_conv_back(rv, Relax{nullptr, 0}, nd.W, nd.b, Mc, g, pg, mode_of(nd.src),
                                                     P[nd.src], net->nodes[nd.src].n, cpart, nullptr, 0.f,
                                                     net->num_sms, s));
                        LAUNCH(net, launch_add_partials(cst, cpart, conv_back_tiles(g), Mc, s));
                        written[nd.src] = 1;
                        break;
                    }
                    case VF_RELU:
                        LAUNCH(net, launch_relax_alpha_rows(P[v], Mc, nv, bd.relax[v], pg, al[v], P[nd.src], cst, s,
                                                            0, written[nd.src] ? 1 : 0, bt[v]));
                        written[nd.src] = 1;
                        break;
                    case VF_ADD:
                        for (int src : {nd.src, nd.src2}) {
                            LAUNCH(net, launch_relax_rows(rv, Relax{nullptr, 0}, Mc, nv, pg, P[src], nv,
                                                          written[src] ? 1 : 0, nullptr, s));
                            written[src] = 1;
                        }
                        break;
                    default:
                        return fail(VF_ERR_ARG, "bad node kind");
                }
            }
            if (!written[0]) return fail(VF_ERR_ARG, "internal: the input was not reached");
            LAUNCH(net, launch_concretize_grad(P[0], Mc, (int)n0, pg, centres, eps, cst, lbc, G[0], s));
            if (it == 0 && lb_start) CU(cudaMemcpyAsync(lb_start + m0, lbc, sizeof(float) * Mc, cudaMemcpyDeviceToDevice, s));
            LAUNCH(net, launch_best_update(lb + m0, lbc, Mc, it == 0 ? 1 : 0, s));
            if (!grad_mode && it == iters) break;
            // ---- up: gradient over every node's output, in topological order
            for (int v = 1; v < L; ++v) {
                const Node& nd = net->nodes[v];
                const int nv = (int)nd.n;
                switch (nd.op) {
                    case VF_DENSE:
                        TRY(fwd_product(net, nd, G[nd.src], Mc, (int)net->nodes[nd.src].n, false, nd.b, G[v], s));
                        break;
                    case VF_CONV2D:
                        LAUNCH(net, launch_ibp_conv(G[nd.src], nullptr, nd.W, nd.Wabs, nd.b, (int)Mc, conv_geom(net, nd),
                                                    G[v], nullptr, s));
                        break;
                    case VF_RELU: {
                        CU(cudaMemcpyAsync(G[v], G[nd.src], sizeof(float) * Mc * nv, cudaMemcpyDeviceToDevice, s));
                        float* gout = grad_mode ? grad_out + aoff[v] + m0 * nv : nullptr;
                        if (written[v]) {
                            LAUNCH(net, launch_relax_grad_adam(G[v], P[v], Mc, nv, bd.relax[v], pg, al[v], gout, M1[v],
                                                               M2[v], grad_mode ? 0 : it + 1, lr, s, bt[v]));
                        } else {  // not an ancestor of the last node: zero gradients
                            if (gout != nullptr) CU(cudaMemsetAsync(gout, 0, sizeof(float) * Mc * nv, s));
                            if (bt[v].grad_out != nullptr)
                                CU(cudaMemsetAsync(bt[v].grad_out, 0, sizeof(float) * Mc * nv, s));
                        }
                        break;
                    }
                    case VF_ADD: {
                        const RowRef r1{G[nd.src], 0, nv, kHugeRows, 0}, r2{G[nd.src2], 0, nv, kHugeRows, 0};
                        LAUNCH(net, launch_relax_rows(r1, Relax{nullptr, 0}, Mc, nv, pg, G[v], nv, 0, nullptr, s));
                        LAUNCH(net, launch_relax_rows(r2, Relax{nullptr, 0}, Mc, nv, pg, G[v], nv, 1, nullptr, s));
                        break;
                    }
                    default:
                        return fail(VF_ERR_ARG, "bad node kind");
                }
            }
        }
        if (!grad_mode && alpha_out)
            for (int u : relus) {
                const long long nu = net->nodes[u].n;
                CU(cudaMemcpyAsync(alpha_out + aoff[u] + m0 * nu, A[u], sizeof(float) * Mc * nu,
                                   cudaMemcpyDeviceToDevice, s));
            }
        if (!grad_mode && o.beta_rows_out)
            for (int u : relus) {
                const long long nu = net->nodes[u].n;
                if (Bt[u] != nullptr)
                    CU(cudaMemcpyAsync(o.beta_rows_out + aoff[u] + m0 * nu, Bt[u], sizeof(float) * Mc * nu,
                                       cudaMemcpyDeviceToDevice, s));
                else
                    CU(cudaMemsetAsync(o.beta_rows_out + aoff[u] + m0 * nu, 0, sizeof(float) * Mc * nu, s));
            }
    }
    return VF_OK;
}

}  // namespace

int vf::set_last_error(int code, const char* msg) {
    g_err = msg;
    return code;
}

// ===================================== C ABI ===============================================

extern "C" {

const char* vf_last_error(void) { return g_err.c_str(); }

int vf_sync(void* stream) {
    CU(cudaStreamSynchronize((cudaStream_t)stream));
    CU(cudaGetLastError());
    return VF_OK;
}

int vf_net_check(vf_net* net) {
    if (net == nullptr) return fail(VF_ERR_ARG, "net is NULL");
    int h = 0;
    CU(cudaMemcpy(&h, net->d_err, sizeof(int), cudaMemcpyDeviceToHost));
    if (h) {
        CU(cudaMemset(net->d_err, 0, sizeof(int)));
        return fail(VF_ERR_TIMEOUT, "a kernel's bounded wait expired; its results were discarded");
    }
    return VF_OK;
}

void vf_net_destroy(vf_net* net) {
    if (net == nullptr) return;
    for (auto& nd : net->nodes) {
        cudaFree(nd.W);
        cudaFree(nd.Wabs);
        cudaFree(nd.b);
        cudaFree(nd.pmW);
        cudaFree(nd.WtHi);
        cudaFree(nd.WtLo);
        cudaFree(nd.WfHi);
        cudaFree(nd.WfLo);
        cudaFree(nd.WaHi);
        cudaFree(nd.WaLo);
        cudaFree(nd.rowsum_abs);
        cudaFree(nd.Wwin);
        cudaFree(nd.Wtc);
        cudaFree(nd.Wtn);
    }
    cudaFree(net->d_err);
    cudaFree(net->ident_row);
    for (auto e : net->ev_free) cudaEventDestroy(e);
    for (auto& p : net->ev_used) {
        cudaEventDestroy(p.e0);
        cudaEventDestroy(p.e1);
    }
    cudaFree(net->ws);
    delete net;
}

static int upload(const float* src, long long count, bool abs_copy, float** out, std::vector<float>& host) {
    host.resize((size_t)count);
    CU(cudaMemcpy(host.data(), src, sizeof(float) * count, cudaMemcpyDefault));
    for (long long i = 0; i < count; ++i)
        if (!std::isfinite(host[i])) return fail(VF_ERR_NONFINITE, "non-finite weight or bias");
    if (abs_copy)
        for (auto& x : host) x = std::fabs(x);
    CU(cudaMalloc(out, sizeof(float) * count));
    CU(cudaMemcpy(*out, host.data(), sizeof(float) * count, cudaMemcpyHostToDevice));
    return VF_OK;
}

static int create_impl(const vf_node_desc* d, int n_nodes, size_t ws_bytes, vf_net* net) {
    CU(cudaGetDevice(&net->device));
    CU(cudaDeviceGetAttribute(&net->num_sms, cudaDevAttrMultiProcessorCount, net->device));
    if (const char* f = getenv("VF_TEST_FAIL_AT")) net->fail_at = atoll(f);
    if (const char* f = getenv("VF_DENSE_KERNEL"))
        net->dense_kernel = (strcmp(f, "ffma") == 0) ? 1 : (strcmp(f, "tc") == 0 ? 2 : 0);
    if (const char* f = getenv("VF_DENSE_TC_MIN_TILES")) net->dense_tc_min_tiles = std::max(0LL, atoll(f));
    if (const char* f = getenv("VF_TEST_TC_STALL")) net->tc_stall = atoi(f) != 0;
    if (const char* f = getenv("VF_CONV_WINDOWS")) net->windows = atoi(f) != 0;
    if (const char* f = getenv("VF_CONV_KERNEL"))
        net->conv_whole_warp = (strcmp(f, "warp") == 0) ? 1 : (strcmp(f, "tile") == 0 ? 0 : 2);
    if (const char* f = getenv("VF_CONV_WIN_KERNEL")) net->conv_win_per_position = (strcmp(f, "1") == 0) ? 1 : 0;
    if (const char* f = getenv("VF_COMPACT")) net->compact = atoi(f) != 0;
    if (const char* f = getenv("VF_CONV_TC")) {
        net->conv_tc = strcmp(f, "0") != 0;
        net->conv_tcn = strcmp(f, "tapn") == 0;
    }
    if (const char* f = getenv("VF_FWD_TC"))
        net->fwd_tc = strcmp(f, "0") == 0 ? 0 : (strcmp(f, "all") == 0 ? 2 : (strcmp(f, "ibp") == 0 ? 3 : 1));
    CU(cudaMalloc(&net->d_err, sizeof(int)));
    CU(cudaMemset(net->d_err, 0, sizeof(int)));
    net->nodes.resize(n_nodes);
    std::vector<float> host;
    for (int v = 0; v < n_nodes; ++v) {
        Node& nd = net->nodes[v];
        const vf_node_desc& x = d[v];
        nd.op = x.op;
        if (v == 0) {
            if (x.op != VF_INPUT) return fail(VF_ERR_ARG, "node 0 must be VF_INPUT");
            if (x.c <= 0 || x.h <= 0 || x.w <= 0) return fail(VF_ERR_SHAPE, "bad input shape");
            nd.c = x.c;
            nd.h = x.h;
            nd.w = x.w;
            nd.n = (long long)x.c * x.h * x.w;
            continue;
        }
        if (x.op == VF_INPUT) return fail(VF_ERR_ARG, "only node 0 may be VF_INPUT");
        if (x.src < 0 || x.src >= v) return fail(VF_ERR_ARG, "node %d: src %d not an earlier node", v, x.src);
        nd.src = x.src;
        const Node& s = net->nodes[x.src];
        net->nodes[x.src].consumers++;
        switch (x.op) {
            case VF_DENSE: {
                if (x.n_out <= 0 || !x.W || !x.b) return fail(VF_ERR_ARG, "node %d: dense needs n_out, W, b", v);
                nd.c = x.n_out;
                nd.h = nd.w = 1;
                nd.n = x.n_out;
                const long long cnt = nd.n * s.n;
                TRY(upload(x.W, cnt, false, &nd.W, host));
                TRY(upload(x.W, cnt, true, &nd.Wabs, host));
                TRY(upload(x.b, nd.n, false, &nd.b, host));
                {  // row sums of |W| (host copy of W is still in `host` from the |W| upload above)
                    std::vector<float> rs((size_t)nd.n, 0.f), wabs((size_t)cnt);
                    CU(cudaMemcpy(wabs.data(), nd.Wabs, sizeof(float) * cnt, cudaMemcpyDeviceToHost));
                    for (long long o = 0; o < nd.n; ++o) {
                        float acc = 0.f;
                        for (long long i = 0; i < s.n; ++i) acc += wabs[o * s.n + i];
                        rs[o] = acc;
                    }
                    CU(cudaMalloc(&nd.rowsum_abs, sizeof(float) * nd.n));
                    CU(cudaMemcpy(nd.rowsum_abs, rs.data(), sizeof(float) * nd.n, cudaMemcpyHostToDevice));
                }
                // [W; -W] for the first step of a pass that starts at this node
                std::vector<float> pm((size_t)(2 * cnt));
                CU(cudaMemcpy(pm.data(), nd.W, sizeof(float) * cnt, cudaMemcpyDeviceToHost));
                for (long long i = 0; i < cnt; ++i) pm[cnt + i] = -pm[i];
                CU(cudaMalloc(&nd.pmW, sizeof(float) * 2 * cnt));
                CU(cudaMemcpy(nd.pmW, pm.data(), sizeof(float) * 2 * cnt, cudaMemcpyHostToDevice));
                if (nd.n % 4 == 0) {  // TMA rows of W^T need a 16-byte stride
                    // 3xTF32 split of W^T: head = fp32 with the 13 low mantissa bits cleared (exact tf32),
                    // remainder = W - head (exact in fp32).
                    const long long nin = s.n, nout = nd.n;
                    std::vector<float> hi((size_t)cnt), lo((size_t)cnt);
                    for (long long o = 0; o < nout; ++o)
                        for (long long i = 0; i < nin; ++i) {
                            const float wv = pm[o * nin + i];
                            uint32_t bits;
                            std::memcpy(&bits, &wv, 4);
                            bits &= 0xFFFFE000u;
                            float h;
                            std::memcpy(&h, &bits, 4);
                            hi[i * nout + o] = h;
                            lo[i * nout + o] = wv - h;
                        }
                    CU(cudaMalloc(&nd.WtHi, sizeof(float) * cnt));
                    CU(cudaMalloc(&nd.WtLo, sizeof(float) * cnt));
                    CU(cudaMemcpy(nd.WtHi, hi.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                    CU(cudaMemcpy(nd.WtLo, lo.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                }
                if (s.n % 4 == 0) {  // TMA rows of W (forward products) need a 16-byte stride
                    std::vector<float> hi((size_t)cnt), lo((size_t)cnt);
                    for (long long i = 0; i < cnt; ++i) {
                        uint32_t bits;
                        std::memcpy(&bits, &pm[i], 4);
                        bits &= 0xFFFFE000u;
                        std::memcpy(&hi[i], &bits, 4);
                        lo[i] = pm[i] - hi[i];
                    }
                    CU(cudaMalloc(&nd.WfHi, sizeof(float) * cnt));
                    CU(cudaMalloc(&nd.WfLo, sizeof(float) * cnt));
                    CU(cudaMemcpy(nd.WfHi, hi.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                    CU(cudaMemcpy(nd.WfLo, lo.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                    for (long long i = 0; i < cnt; ++i) {
                        hi[i] = std::fabs(hi[i]);
                        lo[i] = std::fabs(lo[i]);
                    }
                    CU(cudaMalloc(&nd.WaHi, sizeof(float) * cnt));
                    CU(cudaMalloc(&nd.WaLo, sizeof(float) * cnt));
                    CU(cudaMemcpy(nd.WaHi, hi.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                    CU(cudaMemcpy(nd.WaLo, lo.data(), sizeof(float) * cnt, cudaMemcpyHostToDevice));
                }
                break;
            }
            case VF_CONV2D: {
                if (x.n_out <= 0 || x.k <= 0 || x.stride <= 0 || x.pad < 0 || !x.W || !x.b)
                    return fail(VF_ERR_ARG, "node %d: conv needs n_out, k, stride, pad, W, b", v);
                const int ho = (s.h + 2 * x.pad - x.k) / x.stride + 1;
                const int wo = (s.w + 2 * x.pad - x.k) / x.stride + 1;
                if (ho <= 0 || wo <= 0) return fail(VF_ERR_SHAPE, "node %d: empty conv output", v);
                nd.c = x.n_out;
                nd.h = ho;
                nd.w = wo;
                nd.k = x.k;
                nd.stride = x.stride;
                nd.pad = x.pad;
                nd.n = (long long)nd.c * ho * wo;
                const long long cnt = (long long)x.n_out * s.c * x.k * x.k;
                TRY(upload(x.W, cnt, false, &nd.W, host));
                TRY(upload(x.W, cnt, true, &nd.Wabs, host));
                TRY(upload(x.b, nd.c, false, &nd.b, host));
                ConvGeom g = conv_geom(net, nd);
                {  // tap-major copy [k*k][co][ci_pad] (+4 floats of skew per tap) for the windowed kernel
                    const int cb = win_ci_block(g.ci);
                    const int ci_pad = (g.ci + cb - 1) / cb * cb;
                    const int ts = g.co * ci_pad + 4;
                    std::vector<float> wt((size_t)g.k * g.k * ts, 0.f), w0((size_t)cnt);
                    CU(cudaMemcpy(w0.data(), nd.W, sizeof(float) * cnt, cudaMemcpyDeviceToHost));
                    for (int co = 0; co < g.co; ++co)
                        for (int ci = 0; ci < g.ci; ++ci)
                            for (int p = 0; p < g.k; ++p)
                                for (int q = 0; q < g.k; ++q)
                                    wt[(size_t)(p * g.k + q) * ts + (size_t)co * ci_pad + ci] =
                                        w0[(((size_t)co * g.ci + ci) * g.k + p) * g.k + q];
                    CU(cudaMalloc(&nd.Wwin, sizeof(float) * wt.size()));
                    CU(cudaMemcpy(nd.Wwin, wt.data(), sizeof(float) * wt.size(), cudaMemcpyHostToDevice));
                    nd.ww = WinWeights{nd.Wwin, ts, ci_pad, cb, net->conv_win_per_position};
                }
                if (conv_tc_weights_supported(g)) {  // operand images of the tensor-core kernel
                    std::vector<float> w0((size_t)cnt), wt((size_t)conv_tc_wtc_floats(g));
                    CU(cudaMemcpy(w0.data(), nd.W, sizeof(float) * cnt, cudaMemcpyDeviceToHost));
                    conv_tc_pack_weights(g, w0.data(), wt.data());
                    CU(cudaMalloc(&nd.Wtc, sizeof(float) * wt.size()));
                    CU(cudaMemcpy(nd.Wtc, wt.data(), sizeof(float) * wt.size(), cudaMemcpyHostToDevice));
                    if (const int nwn = conv_tcn_wtn_floats(g)) {  // the taps-in-N operand images
                        std::vector<float> wn((size_t)nwn);
                        conv_tcn_pack_weights(g, w0.data(), wn.data());
                        CU(cudaMalloc(&nd.Wtn, sizeof(float) * wn.size()));
                        CU(cudaMemcpy(nd.Wtn, wn.data(), sizeof(float) * wn.size(), cudaMemcpyHostToDevice));
                    }
                }
                if (!conv_back_supported(g))
                    return fail(VF_ERR_UNSUPPORTED,
                                "node %d: convolution geometry not supported (stride 1/2/4, pad <= k-1, output covered "
                                "by the input, staged tile within shared memory)", v);
                break;
            }
            case VF_RELU:
                nd.c = s.c;
                nd.h = s.h;
                nd.w = s.w;
                nd.n = s.n;
                break;
            case VF_ADD: {
                if (x.src2 < 0 || x.src2 >= v) return fail(VF_ERR_ARG, "node %d: src2 not an earlier node", v);
                const Node& s2 = net->nodes[x.src2];
                if (s2.c != s.c || s2.h != s.h || s2.w != s.w) return fail(VF_ERR_SHAPE, "node %d: add shapes differ", v);
                nd.src2 = x.src2;
                net->nodes[x.src2].consumers++;
                nd.c = s.c;
                nd.h = s.h;
                nd.w = s.w;
                nd.n = s.n;
                break;
            }
            default:
                return fail(VF_ERR_ARG, "node %d: unknown op %d", v, x.op);
        }
    }
    const int last = n_nodes - 1;
    if (net->nodes[last].op != VF_DENSE && net->nodes[last].op != VF_CONV2D)
        return fail(VF_ERR_UNSUPPORTED, "the last node must be dense or conv");
    net->total = 0;
    long long nmax = 0;
    for (auto& nd : net->nodes) {
        net->total += nd.n;
        nmax = std::max(nmax, nd.n);
    }
    {
        std::vector<float4> id((size_t)nmax, make_float4(1.f, 1.f, 0.f, 0.f));
        CU(cudaMalloc(&net->ident_row, sizeof(float4) * nmax));
        CU(cudaMemcpy(net->ident_row, id.data(), sizeof(float4) * nmax, cudaMemcpyHostToDevice));
    }
    net->ws_bytes = ws_bytes ? ws_bytes : (size_t(4) << 30);
    CU(cudaMalloc(&net->ws, net->ws_bytes));
    return VF_OK;
}

int vf_net_create(const vf_node_desc* nodes, int n_nodes, size_t workspace_bytes, vf_net** out_net) {
    if (!nodes || !out_net || n_nodes < 2) return fail(VF_ERR_ARG, "nodes/out_net NULL or fewer than 2 nodes");
    *out_net = nullptr;
    vf_net* net = new vf_net();
    int r = create_impl(nodes, n_nodes, workspace_bytes, net);
    if (r != VF_OK) {
        std::string keep = g_err;
        vf_net_destroy(net);
        g_err = keep;
        return r;
    }
    *out_net = net;
    return VF_OK;
}

int vf_net_node_size(const vf_net* net, int v) {
    if (!net || v < 0 || v >= (int)net->nodes.size()) return -1;
    return (int)net->nodes[v].n;
}

long long vf_net_total_size(const vf_net* net) { return net ? net->total : -1; }

long long vf_launch_count(const vf_net* net) { return net ? net->launches : -1; }

int vf_ibp(vf_net* net, const float* centres, int B, float eps, float* lb_all, float* ub_all, void* stream) {
    TRY(check_net(net));
    if (!centres || !lb_all || !ub_all || B < 0) return fail(VF_ERR_ARG, "NULL pointer or negative B");
    if (!std::isfinite(eps) || eps < 0.f) return fail(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (B == 0) return VF_OK;
    cudaStream_t s = (cudaStream_t)stream;
    Arena ar{net->ws, net->ws_bytes};
    IbpState st;
    TRY(run_ibp(net, centres, B, eps, ar, st, s));
    for (size_t v = 0; v < net->nodes.size(); ++v) {
        const long long off = offset_of(net, (int)v, B);
        LAUNCH(net, launch_bounds_from_cr(st.c[v], st.r[v], (long long)B * net->nodes[v].n, lb_all + off, ub_all + off, s));
    }
    return VF_OK;
}

int vf_crown_backward(vf_net* net, int start_node, const float* lambda0, int R, long long lambda0_bstride,
                      const float* lb_all, const float* ub_all, const float* const* alpha, int B, float* lambda_in,
                      float* const_out, void* stream) {
    TRY(check_net(net));
    if (!lambda0 || !lb_all || !ub_all || !lambda_in || !const_out) return fail(VF_ERR_ARG, "NULL pointer");
    if (start_node < 0 || start_node >= (int)net->nodes.size()) return fail(VF_ERR_ARG, "start_node out of range");
    if (R < 0 || B < 0 || lambda0_bstride < 0) return fail(VF_ERR_ARG, "negative size");
    if (B == 0 || R == 0) return VF_OK;
    cudaStream_t s = (cudaStream_t)stream;
    Arena ar{net->ws, net->ws_bytes};
    const long long n0 = net->nodes[0].n;
    const long long ns = net->nodes[start_node].n;
    if (start_node == 0) {  // nothing to back-substitute
        for (int b = 0; b < B; ++b)
            CU(cudaMemcpyAsync(lambda_in + (long long)b * R * n0, lambda0 + b * lambda0_bstride,
                               sizeof(float) * R * n0, cudaMemcpyDeviceToDevice, s));
        CU(cudaMemsetAsync(const_out, 0, sizeof(float) * B * R, s));
        return VF_OK;
    }
    std::vector<const float*> L(net->nodes.size()), U(net->nodes.size());
    for (size_t v = 0; v < net->nodes.size(); ++v) {
        L[v] = lb_all + offset_of(net, (int)v, B);
        U[v] = ub_all + offset_of(net, (int)v, B);
    }
    std::vector<const float4*> relax;
    TRY(build_relax(net, B, L, U, alpha, ar, relax, s));
    Entry init;
    init.kind = E_VIRT;
    init.ref = RowRef{lambda0, lambda0_bstride, ns, R, 0};
    return run_pass(net, start_node, init, (long long)B * R, R, ar, relax, nullptr, 0.f, nullptr, lambda_in, const_out,
                    s);
}

int vf_concretize(const float* lambda, const float* cst, const float* centres, float eps, int B, int R, int n0,
                  float* lb, void* stream) {
    if (!lambda || !centres || !lb) return fail(VF_ERR_ARG, "NULL pointer");
    if (B < 0 || R < 0 || n0 <= 0) return fail(VF_ERR_ARG, "bad sizes");
    if (!std::isfinite(eps) || eps < 0.f) return fail(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (B == 0 || R == 0) return VF_OK;
    CU(launch_concretize_api(lambda, cst, centres, eps, B, R, n0, lb, (cudaStream_t)stream));
    return VF_OK;
}

// The intermediate alpha options (vf_opts.alpha_inter_iters / alpha_inter_lr) of any call.
int check_inter_opts(const vf_opts& o) {
    if (o.alpha_inter_iters < 0) return fail(VF_ERR_ARG, "alpha_inter_iters must be >= 0");
    if (o.alpha_inter_iters == 0) return VF_OK;
    if (!std::isfinite(o.alpha_inter_lr) || o.alpha_inter_lr < 0.f)
        return fail(VF_ERR_NONFINITE, "alpha_inter_lr must be finite and >= 0");
    if (o.no_host_sync) return fail(VF_ERR_UNSUPPORTED, "intermediate alpha optimisation synchronises the stream");
    if (o.sound) return fail(VF_ERR_UNSUPPORTED, "intermediate alpha optimisation is not part of the sound mode");
    return VF_OK;
}

int vf_verify_batch(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                    const vf_opts* opts, float* lb, float* ub, float* lb_ibp, uint8_t* verified, void* stream) {
    TRY(check_net(net));
    vf_opts o{};
    if (opts) o = *opts;
    TRY(check_inter_opts(o));
    if (!centres || !C || !lb) return fail(VF_ERR_ARG, "centres, C and lb must not be NULL");
    if (o.both_sides && !ub) return fail(VF_ERR_ARG, "both_sides needs ub");
    if (B < 0 || R < 0 || C_bstride < 0) return fail(VF_ERR_ARG, "negative size");
    if (!std::isfinite(eps) || eps < 0.f) return fail(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (B == 0 || R == 0) return VF_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int nn = (int)net->nodes.size();
    const int last = nn - 1;
    const int nL = (int)net->nodes[last].n;
    const long long n0 = net->nodes[0].n;
    const int BC = C_bstride > 0 ? B : 1;
    Arena ar{net->ws, net->ws_bytes};

    int* finite_flag = nullptr;
    if (!o.skip_finite_check && !o.no_host_sync) {
        std::vector<std::pair<const float*, long long>> arrs = {{centres, (long long)B * n0},
                                                                {C, (long long)(BC - 1) * C_bstride + (long long)R * nL}};
        if (o.alpha)
            for (int v = 0; v < nn; ++v)
                if (net->nodes[v].op == VF_RELU && o.alpha[v]) arrs.push_back({o.alpha[v], (long long)B * net->nodes[v].n});
        TRY(scan_finite_dev(net, arrs, ar, s, &finite_flag));
    }

    struct SoundScope {  // contractions take the FFMA kernels (whose rounding the error analysis models)
        vf_net* n;
        SoundScope(vf_net* n_, int on) : n(n_) { n->call_sound = on; }
        ~SoundScope() { n->call_sound = 0; }
    } scope(net, o.sound ? 1 : 0);
    IbpState st;
    Bounds bd;
    TRY(prepare_bounds(net, centres, B, eps, o, ar, st, bd, s, finite_flag));
    if (o.sound) TRY(sound_weights(net, B, eps, centres, st, bd, last, ar, s));
    std::vector<float*>& Lw = bd.Lw;
    std::vector<float*>& Uw = bd.Uw;
    std::vector<const float4*>& relax = bd.relax;
    const int Rp = o.both_sides ? 2 * R : R;
    float* pass_out = ar.take<float>((size_t)B * Rp);
    float* lbI = ar.take<float>((size_t)B * R);
    float* ubI = ar.take<float>((size_t)B * R);
    float* S = o.both_sides ? ar.take<float>((size_t)BC * Rp * nL) : nullptr;
    if (!pass_out || !lbI || !ubI || (o.both_sides && !S)) return fail(VF_ERR_WORKSPACE, "workspace too small");

    // Specification pass.
    Entry init;
    init.kind = E_VIRT;
    if (o.both_sides) {
        LAUNCH(net, launch_spec_rows(C, C_bstride, BC, R, nL, S, s));
        init.ref = RowRef{S, BC > 1 ? (long long)Rp * nL : 0, nL, Rp, 0};
    } else {
        init.ref = RowRef{C, C_bstride, nL, R, 0};
    }
    TRY(run_pass(net, last, init, (long long)B * Rp, Rp, ar, relax, centres, eps, pass_out, nullptr, nullptr, s,
                 nullptr, o.sound ? &bd.sw : nullptr));
    LAUNCH(net, launch_spec_ibp(C, C_bstride, B, R, nL, st.c[last], st.r[last], lbI, ubI, s,
                                o.sound ? gamma_up(2LL * nL + 64) : 0.f));
    LAUNCH(net, launch_decide(lbI, ubI, pass_out, B, R, o.both_sides, lb, ub, lb_ibp, verified, s));

    if (o.pre_lb || o.pre_ub) {
        for (int v = 0; v < nn; ++v) {
            const long long off = offset_of(net, v, B);
            const long long cnt = (long long)B * net->nodes[v].n;
            if (Lw[v]) {
                if (o.pre_lb) CU(cudaMemcpyAsync(o.pre_lb + off, Lw[v], sizeof(float) * cnt, cudaMemcpyDeviceToDevice, s));
                if (o.pre_ub) CU(cudaMemcpyAsync(o.pre_ub + off, Uw[v], sizeof(float) * cnt, cudaMemcpyDeviceToDevice, s));
            } else {
                float* tl = o.pre_lb ? o.pre_lb + off : nullptr;
                float* tu = o.pre_ub ? o.pre_ub + off : nullptr;
                if (tl && tu) LAUNCH(net, launch_bounds_from_cr(st.c[v], st.r[v], cnt, tl, tu, s, nullptr, o.sound ? 1 : 0));
            }
        }
    }
    return VF_OK;
}

int vf_alpha_crown(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                   const vf_opts* opts, int iters, float lr, float* lb, float* lb_start, float* alpha_out,
                   void* stream) {
    TRY(check_net(net));
    vf_opts o{};
    if (opts) o = *opts;
    TRY(check_inter_opts(o));
    if (!centres || !C || !lb) return fail(VF_ERR_ARG, "centres, C and lb must not be NULL");
    if (B < 0 || R < 0 || C_bstride < 0 || iters < 0) return fail(VF_ERR_ARG, "negative size");
    if (!std::isfinite(eps) || eps < 0.f || !std::isfinite(lr) || lr < 0.f)
        return fail(VF_ERR_NONFINITE, "eps and lr must be finite and >= 0");
    if (o.both_sides) return fail(VF_ERR_UNSUPPORTED, "alpha optimisation bounds the lower side; pass -C for upper");
    if (o.sound) return fail(VF_ERR_UNSUPPORTED, "the sound-in-fp32 mode covers vf_verify_batch only");
    if (B == 0 || R == 0) return VF_OK;
    if (!affine_chain(net))
        return spec_alpha_graph(net, centres, B, eps, C, R, C_bstride, o, iters, lr, false, nullptr, nullptr, lb,
                                lb_start, alpha_out, (cudaStream_t)stream);
    return spec_alpha(net, centres, B, eps, C, R, C_bstride, o, iters, lr, false, nullptr, nullptr, lb, lb_start,
                      alpha_out, (cudaStream_t)stream);
}

int vf_alpha_grad(vf_net* net, const float* centres, int B, float eps, const float* C, int R, long long C_bstride,
                  const vf_opts* opts, const float* alpha, float* lb, float* grad, void* stream) {
    return vf_alpha_beta_grad(net, centres, B, eps, C, R, C_bstride, opts, alpha, nullptr, lb, grad, nullptr, stream);
}

int vf_alpha_beta_grad(vf_net* net, const float* centres, int B, float eps, const float* C, int R,
                       long long C_bstride, const vf_opts* opts, const float* alpha, const float* beta, float* lb,
                       float* grad_alpha, float* grad_beta, void* stream) {
    TRY(check_net(net));
    vf_opts o{};
    if (opts) o = *opts;
    TRY(check_inter_opts(o));
    if (!centres || !C || !lb || !alpha || !grad_alpha) return fail(VF_ERR_ARG, "NULL pointer");
    if (B < 0 || R < 0 || C_bstride < 0) return fail(VF_ERR_ARG, "negative size");
    if (!std::isfinite(eps) || eps < 0.f) return fail(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (o.both_sides) return fail(VF_ERR_UNSUPPORTED, "alpha optimisation bounds one side: pass -C for upper bounds");
    if (o.sound) return fail(VF_ERR_UNSUPPORTED, "the sound-in-fp32 mode covers vf_verify_batch only");
    if (B == 0 || R == 0) return VF_OK;
    if (!affine_chain(net))
        return spec_alpha_graph(net, centres, B, eps, C, R, C_bstride, o, 0, 0.f, true, alpha, grad_alpha, lb, nullptr,
                                nullptr, (cudaStream_t)stream, beta, grad_beta);
    return spec_alpha(net, centres, B, eps, C, R, C_bstride, o, 0, 0.f, true, alpha, grad_alpha, lb, nullptr, nullptr,
                      (cudaStream_t)stream, beta, grad_beta);
}

int vf_abi_layout(int which, int field, size_t* out) {
    if (!out) return fail(VF_ERR_ARG, "NULL pointer");
#define VF_OFF(T, f) offsetof(T, f)
    static const size_t node[] = {VF_OFF(vf_node_desc, op),     VF_OFF(vf_node_desc, src), VF_OFF(vf_node_desc, src2),
                                  VF_OFF(vf_node_desc, c),      VF_OFF(vf_node_desc, h),   VF_OFF(vf_node_desc, w),
                                  VF_OFF(vf_node_desc, n_out),  VF_OFF(vf_node_desc, k),   VF_OFF(vf_node_desc, stride),
                                  VF_OFF(vf_node_desc, pad),    VF_OFF(vf_node_desc, W),   VF_OFF(vf_node_desc, b)};
    static const size_t opts[] = {VF_OFF(vf_opts, relu_crown),      VF_OFF(vf_opts, alpha),
                                  VF_OFF(vf_opts, both_sides),      VF_OFF(vf_opts, skip_finite_check),
                                  VF_OFF(vf_opts, pre_lb),          VF_OFF(vf_opts, pre_ub),
                                  VF_OFF(vf_opts, no_host_sync),    VF_OFF(vf_opts, split),
                                  VF_OFF(vf_opts, sound),           VF_OFF(vf_opts, alpha_inter_iters),
                                  VF_OFF(vf_opts, alpha_inter_lr),  VF_OFF(vf_opts, alpha_rows_init),
                                  VF_OFF(vf_opts, beta_rows_init),  VF_OFF(vf_opts, beta_rows_out)};
    static const size_t bopts[] = {VF_OFF(vf_bab_opts, max_domains),       VF_OFF(vf_bab_opts, batch),
                                   VF_OFF(vf_bab_opts, alpha_iters),       VF_OFF(vf_bab_opts, lr),
                                   VF_OFF(vf_bab_opts, relu_crown),        VF_OFF(vf_bab_opts, trace),
                                   VF_OFF(vf_bab_opts, trace_cap),         VF_OFF(vf_bab_opts, alpha_inter_iters),
                                   VF_OFF(vf_bab_opts, alpha_inter_lr),    VF_OFF(vf_bab_opts, cold_start)};
    static const size_t bres[] = {VF_OFF(vf_bab_result, status), VF_OFF(vf_bab_result, domains),
                                  VF_OFF(vf_bab_result, rounds), VF_OFF(vf_bab_result, max_depth),
                                  VF_OFF(vf_bab_result, lb)};
#undef VF_OFF
    const size_t* tab[] = {node, opts, bopts, bres};
    const int count[] = {12, 14, 10, 5};
    const size_t size[] = {sizeof(vf_node_desc), sizeof(vf_opts), sizeof(vf_bab_opts), sizeof(vf_bab_result)};
    if (which < 0 || which > 3 || field < -1 || field >= count[which]) return fail(VF_ERR_ARG, "no such struct field");
    *out = field < 0 ? size[which] : tab[which][field];
    return VF_OK;
}

int vf_net_node_info(const vf_net* net, int v, int* op, int* src, int* src2, long long* n) {
    TRY(check_net(net));
    if (v < 0 || v >= (int)net->nodes.size()) return fail(VF_ERR_ARG, "node index out of range");
    const Node& nd = net->nodes[v];
    if (op) *op = nd.op;
    if (src) *src = nd.src;
    if (src2) *src2 = nd.src2;
    if (n) *n = nd.n;
    return VF_OK;
}

int vf_profile_enable(vf_net* net, int enable) {
    TRY(check_net(net));
    net->prof = enable != 0;
    return VF_OK;
}

int vf_profile_read(vf_net* net, int kind, long long* launches, double* total_ms, double* flops, int reset) {
    TRY(check_net(net));
    if (kind < 0 || kind > 7) return fail(VF_ERR_ARG, "bad kernel kind");
    for (auto& t : net->ev_used) {
        CU(cudaEventSynchronize(t.e1));
        float ms = 0.f;
        CU(cudaEventElapsedTime(&ms, t.e0, t.e1));
        for (int k : {0, t.kind}) {
            net->prof_ms[k] += ms;
            net->prof_launches[k]++;
            net->prof_flops[k] += t.flops;
        }
        net->ev_free.push_back(t.e0);
        net->ev_free.push_back(t.e1);
    }
    net->ev_used.clear();
    if (launches) *launches = net->prof_launches[kind];
    if (total_ms) *total_ms = net->prof_ms[kind];
    if (flops) *flops = net->prof_flops[kind];
    if (reset)
        for (int k = 0; k < 8; ++k) {
            net->prof_launches[k] = 0;
            net->prof_ms[k] = 0.0;
            net->prof_flops[k] = 0.0;
        }
    return VF_OK;
}

}  // extern "C"
