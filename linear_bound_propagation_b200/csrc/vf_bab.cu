// Branch and bound over ReLU splits (vf_bab_verify): the search on the host, every bound and every
// per-subdomain decision on the device.
//
// Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully Sharded Data
// Parallelism", technical summary §2.2, §3 and §4.3 (complete verification by beta-CROWN with
// branch-and-bound; the page names the method only). The search is one plain best-first reading:
// bound the whole box; while some subdomain is open, take the open ones with the lowest bound (a batch
// of them), split each on its highest-scoring unstable neuron into z <= 0 and z >= 0, and bound all
// children in one batched vf_verify_batch + vf_alpha_crown call (the split multipliers beta are
// optimised with the slopes). A child closes when its bounds contradict (no input) or all its rows are
// positive; a child with nothing left to split ends the search undecided.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <utility>
#include <vector>

#include "vf.h"
#include "vf_internal.cuh"

namespace {

using vf::BabPick;

// Scratch of one search, stream-ordered: allocated from the device's memory pool on the search's stream and
// released on it when the buffer goes out of scope, after the work queued on that stream (no device-wide
// synchronisation, as a plain free would take).
struct DeviceBuffer {
    void* p = nullptr;
    cudaStream_t s = nullptr;
    DeviceBuffer() = default;
    DeviceBuffer(const DeviceBuffer&) = delete;
    DeviceBuffer& operator=(const DeviceBuffer&) = delete;
    ~DeviceBuffer() {
        if (p) cudaFreeAsync(p, s);
    }
    cudaError_t alloc(size_t bytes, cudaStream_t stream) {
        s = stream;
        return cudaMallocAsync(&p, bytes, stream);
    }
    template <class T>
    T* get() const {
        return static_cast<T*>(p);
    }
};

int cuda_fail(cudaError_t e, const char* what) {
    char buf[256];
    snprintf(buf, sizeof buf, "%s: %s", what, cudaGetErrorString(e));
    return vf::set_last_error(VF_ERR_CUDA, buf);
}

#define BAB_CU(x)                                    \
    do {                                             \
        cudaError_t e_ = (x);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, #x); \
    } while (0)
#define BAB_TRY(x)               \
    do {                         \
        int r_ = (x);            \
        if (r_ != VF_OK) return r_; \
    } while (0)

// One subdomain: its split constraints (search-wide neuron index, sign), lowest row bound, creation
// number and the neuron it will be split on.
struct Domain {
    float lb;
    long long seq;
    std::vector<std::pair<int, signed char>> splits;
    int branch;
};

struct ReluLayer {
    int node;       // the ReLU node
    long long off;  // offset of its input node's block per centre row in the vf_ibp layout
    int n;          // neurons
    int gbase;      // search-wide index of its first neuron
};

// Everything the device bound function needs: the handle, the options, and the round's buffers.
struct DeviceBound {
    vf_net* net;
    const vf_bab_opts* opts;
    float eps;
    const float* C;
    int R;
    void* stream;
    int nn, sum_n;
    const std::vector<ReluLayer>* layers;
    float *cen, *lbv, *lba, *plb, *pub;
    signed char* spl;
    BabPick* pick;
    const long long* meta_off;
    const int *meta_n, *meta_g;
    std::vector<signed char> hsplit;
    std::vector<BabPick> hpick;
    long long traced = 0;  // entries of opts->trace written so far
    // warm starts: each bounded subdomain's last slopes and multipliers in a pool slot, found by its split list
    bool warm = false;
    int pool_cap = 0;
    float *pool_a = nullptr, *pool_b = nullptr;  // [pool_cap, R, sum_n]
    float *init_a, *init_b, *out_a, *out_b;      // [D, R, sum_n] in the alpha_out layout of a batch
    int* dslots = nullptr;                       // [2 D]: parents' slots, then the children's
    std::map<std::vector<int>, int> slot_of;
    std::vector<int> free_slots;
    int next_slot = 0;
};

// vf_bab_bound_fn on the device: one vf_verify_batch (bounds and pre-activation bounds of all n subdomains
// with their split constraints) and, with alpha_iters, one vf_alpha_crown (slopes and split multipliers),
// then bab_pick_k and one copy back.
int device_bound(void* user, int n, const int* split_offset, const int* split_count, const int* split_neuron,
                 const signed char* split_sign, float* lb, int* branch, int* empty) {
    DeviceBound& d = *static_cast<DeviceBound*>(user);
    const std::vector<ReluLayer>& layers = *d.layers;
    const int nl = (int)layers.size();
    cudaStream_t s = (cudaStream_t)d.stream;
    d.hsplit.assign((size_t)n * d.sum_n, 0);
    for (int i = 0; i < n; ++i)
        for (int k = 0; k < split_count[i]; ++k) {
            const int g = split_neuron[split_offset[i] + k];
            int q = 0;
            while (q + 1 < nl && layers[q + 1].gbase <= g) ++q;
            if (g < layers[q].gbase || g >= layers[q].gbase + layers[q].n)
                return vf::set_last_error(VF_ERR_ARG, "split neuron index out of range");
            d.hsplit[(size_t)n * layers[q].gbase + (size_t)i * layers[q].n + (g - layers[q].gbase)] =
                split_sign[split_offset[i] + k];
        }
    if (d.sum_n > 0) BAB_CU(cudaMemcpyAsync(d.spl, d.hsplit.data(), d.hsplit.size(), cudaMemcpyHostToDevice, s));
    std::vector<const signed char*> sp(d.nn, nullptr);
    for (const auto& L : layers) sp[L.node] = d.spl + (size_t)n * L.gbase;
    vf_opts o{};
    o.relu_crown = d.opts->relu_crown;
    o.split = sp.data();
    o.pre_lb = d.plb;
    o.pre_ub = d.pub;
    o.alpha_inter_iters = d.opts->alpha_inter_iters;
    o.alpha_inter_lr = d.opts->alpha_inter_lr;
    BAB_TRY(vf_verify_batch(d.net, d.cen, n, d.eps, d.C, d.R, 0, &o, d.lbv, nullptr, nullptr, nullptr, d.stream));
    if (d.opts->alpha_iters > 0) {
        vf_opts oa{};
        oa.relu_crown = d.opts->relu_crown;
        oa.split = sp.data();
        oa.alpha_inter_iters = d.opts->alpha_inter_iters;
        oa.alpha_inter_lr = d.opts->alpha_inter_lr;
        std::vector<int> slots(2 * (size_t)n, -1), keyv;
        std::vector<std::vector<int>> keys(n);
        if (d.warm) {
            // a child's splits are its parent's followed by one more: the parent's key drops the last entry
            for (int i = 0; i < n; ++i) {
                for (int k = 0; k < split_count[i]; ++k)
                    keys[i].push_back(2 * split_neuron[split_offset[i] + k] + (split_sign[split_offset[i] + k] > 0));
                if (!keys[i].empty()) {
                    keyv.assign(keys[i].begin(), keys[i].end() - 1);
                    auto it = d.slot_of.find(keyv);
                    if (it != d.slot_of.end()) slots[i] = it->second;
                }
                if (!d.free_slots.empty()) {
                    slots[n + i] = d.free_slots.back();
                    d.free_slots.pop_back();
                } else if (d.next_slot < d.pool_cap) {
                    slots[n + i] = d.next_slot++;
                }
            }
            BAB_CU(cudaMemcpyAsync(d.dslots, slots.data(), sizeof(int) * 2 * n, cudaMemcpyHostToDevice, s));
            BAB_CU(vf::launch_bab_state(d.pool_a, d.dslots, n, d.R, d.sum_n, d.meta_n, d.meta_g, nl, d.init_a, 0, s));
            BAB_CU(vf::launch_bab_state(d.pool_b, d.dslots, n, d.R, d.sum_n, d.meta_n, d.meta_g, nl, d.init_b, 0, s));
            oa.alpha_rows_init = d.init_a;
            oa.beta_rows_init = d.init_b;
            oa.beta_rows_out = d.out_b;
        }
        BAB_TRY(vf_alpha_crown(d.net, d.cen, n, d.eps, d.C, d.R, 0, &oa, d.opts->alpha_iters, d.opts->lr, d.lba, nullptr,
                               d.warm ? d.out_a : nullptr, d.stream));
        if (d.warm) {
            BAB_CU(vf::launch_bab_state(d.pool_a, d.dslots + n, n, d.R, d.sum_n, d.meta_n, d.meta_g, nl, d.out_a, 1, s));
            BAB_CU(vf::launch_bab_state(d.pool_b, d.dslots + n, n, d.R, d.sum_n, d.meta_n, d.meta_g, nl, d.out_b, 1, s));
            // both children of a parent are bounded in the same round: its slot is free again (the copies above
            // are ordered before any later gather or scatter on the stream)
            for (int i = 0; i < n; ++i) {
                if (!keys[i].empty()) {
                    keyv.assign(keys[i].begin(), keys[i].end() - 1);
                    auto it = d.slot_of.find(keyv);
                    if (it != d.slot_of.end()) {
                        d.free_slots.push_back(it->second);
                        d.slot_of.erase(it);
                    }
                }
                if (slots[n + i] >= 0) d.slot_of[keys[i]] = slots[n + i];
            }
        }
    }
    BAB_CU(vf::launch_bab_pick(d.plb, d.pub, n, d.meta_off, d.meta_n, d.meta_g, nl, d.lbv,
                               d.opts->alpha_iters > 0 ? d.lba : nullptr, d.R, d.pick, s));
    BAB_CU(cudaMemcpyAsync(d.hpick.data(), d.pick, sizeof(BabPick) * n, cudaMemcpyDeviceToHost, s));
    BAB_CU(cudaStreamSynchronize(s));
    for (int i = 0; i < n; ++i) {
        lb[i] = d.hpick[i].minlb;
        branch[i] = d.hpick[i].best;
        empty[i] = d.hpick[i].empty;
        if (d.opts->trace != nullptr && d.traced < d.opts->trace_cap) d.opts->trace[d.traced++] = branch[i];
    }
    return VF_OK;
}

}  // namespace

extern "C" int vf_bab_verify(vf_net* net, const float* centre, float eps, const float* C, int R,
                             const vf_bab_opts* opts, vf_bab_result* result, void* stream) {
    if (!net || !centre || !C || !opts || !result) return vf::set_last_error(VF_ERR_ARG, "NULL pointer");
    if (R <= 0) return vf::set_last_error(VF_ERR_ARG, "R must be positive");
    if (opts->max_domains < 1 || opts->batch < 2 || opts->batch % 2 != 0 || opts->alpha_iters < 0)
        return vf::set_last_error(VF_ERR_ARG, "need max_domains >= 1, an even batch >= 2 and alpha_iters >= 0");
    if (!std::isfinite(eps) || eps < 0.f) return vf::set_last_error(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (!std::isfinite(opts->lr)) return vf::set_last_error(VF_ERR_NONFINITE, "lr must be finite");
    if (opts->alpha_inter_iters < 0) return vf::set_last_error(VF_ERR_ARG, "alpha_inter_iters must be >= 0");
    cudaStream_t s = (cudaStream_t)stream;

    // ---- the graph: ReLU layers, their input blocks and search-wide neuron indices
    std::vector<long long> node_off;
    int nn = 0;
    long long acc = 0;
    while (vf_net_node_size(net, nn) >= 0) {
        node_off.push_back(acc);
        acc += vf_net_node_size(net, nn);
        ++nn;
    }
    const long long total = vf_net_total_size(net);
    const long long n0 = vf_net_node_size(net, 0);
    std::vector<ReluLayer> layers;
    int sum_n = 0;
    for (int v = 0; v < nn; ++v) {
        int op = 0, src = 0;
        long long n = 0;
        BAB_TRY(vf_net_node_info(net, v, &op, &src, nullptr, &n));
        if (op != VF_RELU) continue;
        layers.push_back(ReluLayer{v, node_off[src], (int)n, sum_n});
        sum_n += (int)n;
    }
    const int D = opts->batch;
    const int nl = (int)layers.size();

    // ---- device buffers for one round of D subdomains
    DeviceBuffer cen, spl, lbv, lba, plb, pub, pick, meta_off, meta_n, meta_g;
    BAB_CU(cen.alloc(sizeof(float) * (size_t)D * n0, s));
    BAB_CU(spl.alloc((size_t)D * std::max(sum_n, 1), s));
    BAB_CU(lbv.alloc(sizeof(float) * (size_t)D * R, s));
    BAB_CU(lba.alloc(sizeof(float) * (size_t)D * R, s));
    BAB_CU(plb.alloc(sizeof(float) * (size_t)D * total, s));
    BAB_CU(pub.alloc(sizeof(float) * (size_t)D * total, s));
    BAB_CU(pick.alloc(sizeof(BabPick) * (size_t)D, s));
    BAB_CU(meta_off.alloc(sizeof(long long) * std::max(nl, 1), s));
    BAB_CU(meta_n.alloc(sizeof(int) * std::max(nl, 1), s));
    BAB_CU(meta_g.alloc(sizeof(int) * std::max(nl, 1), s));
    {
        std::vector<long long> ho(nl);
        std::vector<int> hn(nl), hg(nl);
        for (int q = 0; q < nl; ++q) {
            ho[q] = layers[q].off;
            hn[q] = layers[q].n;
            hg[q] = layers[q].gbase;
        }
        if (nl > 0) {
            BAB_CU(cudaMemcpyAsync(meta_off.p, ho.data(), sizeof(long long) * nl, cudaMemcpyHostToDevice, s));
            BAB_CU(cudaMemcpyAsync(meta_n.p, hn.data(), sizeof(int) * nl, cudaMemcpyHostToDevice, s));
            BAB_CU(cudaMemcpyAsync(meta_g.p, hg.data(), sizeof(int) * nl, cudaMemcpyHostToDevice, s));
        }
    }
    BAB_CU(vf::launch_repeat_row(centre, n0, D, cen.get<float>(), s));

    // ---- 1. candidate counterexamples: the centre, then every row's CROWN minimiser vertex of the box.
    // A negative row at a point is a rounded evaluation: it counts only when the sound mode's upper bound
    // there (both sides, eps = 0), which the exact value C f(x) on the fp32 weights cannot exceed, is < 0.
    auto falsified_at = [&](const float* xs, int P, float* ymin_out, bool* hit) -> int {
        *hit = false;
        DeviceBuffer y, yub;
        BAB_CU(y.alloc(sizeof(float) * (size_t)P * R, s));
        BAB_CU(yub.alloc(sizeof(float) * (size_t)P * R, s));
        vf_opts o{};
        o.relu_crown = opts->relu_crown;
        BAB_TRY(vf_verify_batch(net, xs, P, 0.f, C, R, 0, &o, y.get<float>(), nullptr, nullptr, nullptr, stream));
        std::vector<float> h((size_t)P * R);
        BAB_CU(cudaMemcpyAsync(h.data(), y.p, sizeof(float) * h.size(), cudaMemcpyDeviceToHost, s));
        BAB_CU(cudaStreamSynchronize(s));
        *ymin_out = *std::min_element(h.begin(), h.end());
        if (!(*ymin_out < 0.f)) return VF_OK;
        vf_opts so = o;
        so.both_sides = 1;
        so.sound = 1;
        BAB_TRY(vf_verify_batch(net, xs, P, 0.f, C, R, 0, &so, y.get<float>(), yub.get<float>(), nullptr, nullptr,
                                stream));
        BAB_CU(cudaMemcpyAsync(h.data(), yub.p, sizeof(float) * h.size(), cudaMemcpyDeviceToHost, s));
        BAB_CU(cudaStreamSynchronize(s));
        *hit = *std::min_element(h.begin(), h.end()) < 0.f;
        return VF_OK;
    };
    {
        float ymin = 0.f;
        bool hit = false;
        BAB_TRY(falsified_at(cen.get<float>(), 1, &ymin, &hit));
        if (hit) {
            *result = vf_bab_result{VF_BAB_FALSIFIED, 0, 0, 0, ymin};
            return VF_OK;
        }
    }
    {
        // the whole box's bounds (no split); only a row the box does not already prove positive can fall below
        // 0 at its vertex, so the attack is skipped when every row's bound is > 0
        vf_opts o{};
        o.relu_crown = opts->relu_crown;
        o.pre_lb = plb.get<float>();
        o.pre_ub = pub.get<float>();
        BAB_TRY(vf_verify_batch(net, cen.get<float>(), 1, eps, C, R, 0, &o, lbv.get<float>(), nullptr, nullptr, nullptr,
                                stream));
        std::vector<float> h(R);
        BAB_CU(cudaMemcpyAsync(h.data(), lbv.p, sizeof(float) * R, cudaMemcpyDeviceToHost, s));
        BAB_CU(cudaStreamSynchronize(s));
        if (!(*std::min_element(h.begin(), h.end()) > 0.f)) {
            DeviceBuffer lam, cst, xs;
            BAB_CU(lam.alloc(sizeof(float) * (size_t)R * n0, s));
            BAB_CU(cst.alloc(sizeof(float) * (size_t)R, s));
            BAB_CU(xs.alloc(sizeof(float) * (size_t)R * n0, s));
            BAB_TRY(vf_crown_backward(net, nn - 1, C, R, 0, plb.get<float>(), pub.get<float>(), nullptr, 1,
                                      lam.get<float>(), cst.get<float>(), stream));
            BAB_CU(vf::launch_minimiser_points(centre, lam.get<float>(), eps, n0, R, xs.get<float>(), s));
            float ymin = 0.f;
            bool hit = false;
            BAB_TRY(falsified_at(xs.get<float>(), R, &ymin, &hit));
            if (hit) {
                *result = vf_bab_result{VF_BAB_FALSIFIED, 0, 0, 0, ymin};
                return VF_OK;
            }
        }
    }

    // ---- bound a batch of subdomains on the device; one host synchronisation
    DeviceBound db;
    db.net = net;
    db.opts = opts;
    db.eps = eps;
    db.C = C;
    db.R = R;
    db.stream = stream;
    db.nn = nn;
    db.sum_n = sum_n;
    db.layers = &layers;
    db.cen = cen.get<float>();
    db.spl = spl.get<signed char>();
    db.lbv = lbv.get<float>();
    db.lba = lba.get<float>();
    db.plb = plb.get<float>();
    db.pub = pub.get<float>();
    db.pick = pick.get<BabPick>();
    db.meta_off = meta_off.get<long long>();
    db.meta_n = meta_n.get<int>();
    db.meta_g = meta_g.get<int>();
    db.hpick.resize(D);
    DeviceBuffer pool_a, pool_b, init_a, init_b, out_a, out_b, dslots;
    db.warm = opts->alpha_iters > 0 && !opts->cold_start && sum_n > 0;
    if (db.warm) {
        const size_t per = (size_t)R * sum_n;  // floats of one subdomain's slopes (and of its multipliers)
        const size_t cap_mem = (size_t(1) << 30) / (2 * per * sizeof(float));
        db.pool_cap = (int)std::min<size_t>((size_t)opts->max_domains, cap_mem);
        BAB_CU(pool_a.alloc(sizeof(float) * per * std::max(db.pool_cap, 1), s));
        BAB_CU(pool_b.alloc(sizeof(float) * per * std::max(db.pool_cap, 1), s));
        BAB_CU(init_a.alloc(sizeof(float) * per * D, s));
        BAB_CU(init_b.alloc(sizeof(float) * per * D, s));
        BAB_CU(out_a.alloc(sizeof(float) * per * D, s));
        BAB_CU(out_b.alloc(sizeof(float) * per * D, s));
        BAB_CU(dslots.alloc(sizeof(int) * 2 * D, s));
        db.pool_a = pool_a.get<float>();
        db.pool_b = pool_b.get<float>();
        db.init_a = init_a.get<float>();
        db.init_b = init_b.get<float>();
        db.out_a = out_a.get<float>();
        db.out_b = out_b.get<float>();
        db.dslots = dslots.get<int>();
    }
    return vf_bab_search(device_bound, &db, opts->max_domains, opts->batch, result);
}

extern "C" int vf_bab_search(vf_bab_bound_fn bound, void* user, int max_domains, int batch, vf_bab_result* result) {
    if (!bound || !result) return vf::set_last_error(VF_ERR_ARG, "NULL pointer");
    if (max_domains < 1 || batch < 2 || batch % 2 != 0)
        return vf::set_last_error(VF_ERR_ARG, "need max_domains >= 1 and an even batch >= 2");
    using Splits = std::vector<std::pair<int, signed char>>;
    std::vector<int> off, cnt, nid, br(batch), em(batch);
    std::vector<signed char> sg;
    std::vector<float> lb(batch);
    auto evaluate = [&](const std::vector<const Splits*>& doms) -> int {
        off.clear();
        cnt.clear();
        nid.clear();
        sg.clear();
        for (const Splits* d : doms) {
            off.push_back((int)nid.size());
            cnt.push_back((int)d->size());
            for (const auto& p : *d) {
                nid.push_back(p.first);
                sg.push_back(p.second);
            }
        }
        nid.push_back(0);  // keep the arrays non-empty
        sg.push_back(0);
        return bound(user, (int)doms.size(), off.data(), cnt.data(), nid.data(), sg.data(), lb.data(), br.data(),
                     em.data());
    };

    // ---- 2. the whole box
    const Splits none;
    BAB_TRY(evaluate({&none}));
    if (lb[0] > 0.f) {
        *result = vf_bab_result{VF_BAB_VERIFIED, 1, 0, 0, INFINITY};
        return VF_OK;
    }
    if (br[0] < 0) {
        *result = vf_bab_result{VF_BAB_UNKNOWN, 1, 0, 0, lb[0]};
        return VF_OK;
    }
    std::vector<Domain> open;
    open.push_back(Domain{lb[0], 0, {}, br[0]});
    long long domains = 1, seq = 1;
    int rounds = 0, depth = 0;

    // ---- 3-5. rounds of splitting
    while (!open.empty()) {
        const long long take =
            std::min<long long>({(long long)open.size(), (long long)batch / 2, (max_domains - domains) / 2});
        if (take <= 0) break;
        std::sort(open.begin(), open.end(),
                  [](const Domain& a, const Domain& b) { return a.lb < b.lb || (a.lb == b.lb && a.seq < b.seq); });
        std::vector<Domain> parents(open.begin(), open.begin() + take);
        open.erase(open.begin(), open.begin() + take);
        std::vector<Splits> children;
        children.reserve(2 * take);
        for (const Domain& p : parents)
            for (signed char sign : {(signed char)-1, (signed char)1}) {
                children.push_back(p.splits);
                children.back().push_back({p.branch, sign});
            }
        std::vector<const Splits*> ptrs;
        for (const auto& c : children) ptrs.push_back(&c);
        BAB_TRY(evaluate(ptrs));
        domains += (long long)children.size();
        ++rounds;
        for (size_t i = 0; i < children.size(); ++i) {
            depth = std::max(depth, (int)children[i].size());
            const long long num = seq++;
            if (em[i] || lb[i] > 0.f) continue;
            if (br[i] < 0) {
                *result = vf_bab_result{VF_BAB_UNKNOWN, domains, rounds, depth, lb[i]};
                return VF_OK;
            }
            open.push_back(Domain{lb[i], num, std::move(children[i]), br[i]});
        }
    }
    if (open.empty()) {
        *result = vf_bab_result{VF_BAB_VERIFIED, domains, rounds, depth, INFINITY};
        return VF_OK;
    }
    float worst = INFINITY;
    for (const Domain& d : open) worst = std::min(worst, d.lb);
    *result = vf_bab_result{VF_BAB_UNKNOWN, domains, rounds, depth, worst};
    return VF_OK;
}
