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
#include <utility>
#include <vector>

#include "vf.h"
#include "vf_internal.cuh"

namespace {

using vf::BabPick;

struct DeviceBuffer {
    void* p = nullptr;
    DeviceBuffer() = default;
    DeviceBuffer(const DeviceBuffer&) = delete;
    DeviceBuffer& operator=(const DeviceBuffer&) = delete;
    ~DeviceBuffer() {
        if (p) cudaFree(p);
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

}  // namespace

extern "C" int vf_bab_verify(vf_net* net, const float* centre, float eps, const float* C, int R,
                             const vf_bab_opts* opts, vf_bab_result* result, void* stream) {
    if (!net || !centre || !C || !opts || !result) return vf::set_last_error(VF_ERR_ARG, "NULL pointer");
    if (R <= 0) return vf::set_last_error(VF_ERR_ARG, "R must be positive");
    if (opts->max_domains < 1 || opts->batch < 2 || opts->batch % 2 != 0 || opts->alpha_iters < 0)
        return vf::set_last_error(VF_ERR_ARG, "need max_domains >= 1, an even batch >= 2 and alpha_iters >= 0");
    if (!std::isfinite(eps) || eps < 0.f) return vf::set_last_error(VF_ERR_NONFINITE, "eps must be finite and >= 0");
    if (!std::isfinite(opts->lr)) return vf::set_last_error(VF_ERR_NONFINITE, "lr must be finite");
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
    BAB_CU(cudaMalloc(&cen.p, sizeof(float) * (size_t)D * n0));
    BAB_CU(cudaMalloc(&spl.p, (size_t)D * std::max(sum_n, 1)));
    BAB_CU(cudaMalloc(&lbv.p, sizeof(float) * (size_t)D * R));
    BAB_CU(cudaMalloc(&lba.p, sizeof(float) * (size_t)D * R));
    BAB_CU(cudaMalloc(&plb.p, sizeof(float) * (size_t)D * total));
    BAB_CU(cudaMalloc(&pub.p, sizeof(float) * (size_t)D * total));
    BAB_CU(cudaMalloc(&pick.p, sizeof(BabPick) * (size_t)D));
    BAB_CU(cudaMalloc(&meta_off.p, sizeof(long long) * std::max(nl, 1)));
    BAB_CU(cudaMalloc(&meta_n.p, sizeof(int) * std::max(nl, 1)));
    BAB_CU(cudaMalloc(&meta_g.p, sizeof(int) * std::max(nl, 1)));
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

    // ---- 1. the centre itself
    {
        vf_opts o{};
        o.relu_crown = opts->relu_crown;
        BAB_TRY(vf_verify_batch(net, cen.get<float>(), 1, 0.f, C, R, 0, &o, lbv.get<float>(), nullptr, nullptr, nullptr,
                                stream));
        std::vector<float> y(R);
        BAB_CU(cudaMemcpyAsync(y.data(), lbv.p, sizeof(float) * R, cudaMemcpyDeviceToHost, s));
        BAB_CU(cudaStreamSynchronize(s));
        const float ymin = *std::min_element(y.begin(), y.end());
        if (ymin < 0.f) {
            *result = vf_bab_result{VF_BAB_FALSIFIED, 0, 0, 0, ymin};
            return VF_OK;
        }
    }

    // ---- bound a batch of subdomains; one host synchronisation
    std::vector<signed char> hsplit;
    std::vector<BabPick> hpick(D);
    auto evaluate = [&](const std::vector<const std::vector<std::pair<int, signed char>>*>& doms) -> int {
        const int Dn = (int)doms.size();
        hsplit.assign((size_t)Dn * sum_n, 0);
        for (int i = 0; i < Dn; ++i)
            for (const auto& gs : *doms[i]) {
                int q = 0;
                while (q + 1 < nl && layers[q + 1].gbase <= gs.first) ++q;
                const int j = gs.first - layers[q].gbase;
                hsplit[(size_t)Dn * layers[q].gbase + (size_t)i * layers[q].n + j] = gs.second;
            }
        if (sum_n > 0)
            BAB_CU(cudaMemcpyAsync(spl.p, hsplit.data(), hsplit.size(), cudaMemcpyHostToDevice, s));
        std::vector<const signed char*> sp(nn, nullptr);
        for (const auto& L : layers) sp[L.node] = spl.get<signed char>() + (size_t)Dn * L.gbase;
        vf_opts o{};
        o.relu_crown = opts->relu_crown;
        o.split = sp.data();
        o.pre_lb = plb.get<float>();
        o.pre_ub = pub.get<float>();
        BAB_TRY(vf_verify_batch(net, cen.get<float>(), Dn, eps, C, R, 0, &o, lbv.get<float>(), nullptr, nullptr, nullptr,
                                stream));
        if (opts->alpha_iters > 0) {
            vf_opts oa{};
            oa.relu_crown = opts->relu_crown;
            oa.split = sp.data();
            BAB_TRY(vf_alpha_crown(net, cen.get<float>(), Dn, eps, C, R, 0, &oa, opts->alpha_iters, opts->lr,
                                   lba.get<float>(), nullptr, nullptr, stream));
        }
        BAB_CU(vf::launch_bab_pick(plb.get<float>(), pub.get<float>(), Dn, meta_off.get<long long>(), meta_n.get<int>(),
                                   meta_g.get<int>(), nl, lbv.get<float>(),
                                   opts->alpha_iters > 0 ? lba.get<float>() : nullptr, R, pick.get<BabPick>(), s));
        BAB_CU(cudaMemcpyAsync(hpick.data(), pick.p, sizeof(BabPick) * Dn, cudaMemcpyDeviceToHost, s));
        BAB_CU(cudaStreamSynchronize(s));
        return VF_OK;
    };

    // ---- 2. the whole box
    const std::vector<std::pair<int, signed char>> none;
    BAB_TRY(evaluate({&none}));
    if (hpick[0].minlb > 0.f) {
        *result = vf_bab_result{VF_BAB_VERIFIED, 1, 0, 0, INFINITY};
        return VF_OK;
    }
    if (hpick[0].best < 0) {
        *result = vf_bab_result{VF_BAB_UNKNOWN, 1, 0, 0, hpick[0].minlb};
        return VF_OK;
    }
    std::vector<Domain> open;
    open.push_back(Domain{hpick[0].minlb, 0, {}, hpick[0].best});
    long long domains = 1, seq = 1;
    int rounds = 0, depth = 0;

    // ---- 3-5. rounds of splitting
    while (!open.empty()) {
        const long long take = std::min<long long>({(long long)open.size(), (long long)D / 2,
                                                    (opts->max_domains - domains) / 2});
        if (take <= 0) break;
        std::sort(open.begin(), open.end(),
                  [](const Domain& a, const Domain& b) { return a.lb < b.lb || (a.lb == b.lb && a.seq < b.seq); });
        std::vector<Domain> parents(open.begin(), open.begin() + take);
        open.erase(open.begin(), open.begin() + take);
        std::vector<std::vector<std::pair<int, signed char>>> children;
        children.reserve(2 * take);
        for (const Domain& p : parents)
            for (signed char sign : {(signed char)-1, (signed char)1}) {
                children.push_back(p.splits);
                children.back().push_back({p.branch, sign});
            }
        std::vector<const std::vector<std::pair<int, signed char>>*> ptrs;
        for (const auto& c : children) ptrs.push_back(&c);
        BAB_TRY(evaluate(ptrs));
        domains += (long long)children.size();
        ++rounds;
        for (size_t i = 0; i < children.size(); ++i) {
            depth = std::max(depth, (int)children[i].size());
            const long long num = seq++;
            const BabPick& pk = hpick[i];
            if (pk.empty || pk.minlb > 0.f) continue;
            if (pk.best < 0) {
                *result = vf_bab_result{VF_BAB_UNKNOWN, domains, rounds, depth, pk.minlb};
                return VF_OK;
            }
            open.push_back(Domain{pk.minlb, num, std::move(children[i]), pk.best});
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
