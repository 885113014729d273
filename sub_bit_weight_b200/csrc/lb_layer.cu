// Layer objects, their private weight layouts, execution plans and stacks.
//
// A layer is built from the canonical packed signs (one bit per sign, sign(0)
// = +1) and binary16 scales of its two paths (LittleBit notes page,
// "Multi-scale compensation" and "Residual compensation").  It re-tiles the
// signs into the layouts its kernels stream (see lb_internal.cuh) and keeps
// the scales zero-padded, so padded rank slots and rows contribute nothing.

#include <algorithm>
#include <array>
#include <map>
#include <mutex>
#include <cstring>
#include <new>

#include "lb_attr_cache.h"
#include "lb_prefill.cuh"

namespace lb {

__device__ __forceinline__ uint32_t canon_bit(const uint32_t *P, int wpr, int64_t row, int col)
{
    return (__ldg(P + row * wpr + (col >> 5)) >> (col & 31)) & 1u;
}

// Contraction-1 tiles: rows are latent indices of both paths (path p owns
// rows [p*r16, p*r16 + r16)), k runs over the K inputs.  Bit = V_sign[k][j] < 0.
__global__ void build_vtiles_kernel(uint2 *__restrict__ vt, int RG1, int KB1e, int r, int r16, int K,
                                    int npaths, const uint32_t *__restrict__ V0,
                                    const uint32_t *__restrict__ V1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RG1 * KB1e * 32;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t u = idx >> 5;
        const int kb = (int)(u % KB1e);
        const int rg = (int)(u / KB1e);
        const int g = lane >> 2, t = lane & 3;
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int row = rg * kRowsPerGroup + 16 * (i & 3) + g + 8 * (i >> 2);
                    const int k = kb * kKPerBlock + 4 * t + b + 16 * q;
                    const int p = row / r16;
                    const int j = row - p * r16;
                    if (p < npaths && j < r && k < K)
                        w[q] |= canon_bit(p ? V1 : V0, wpr, k, j) << (8 * b + i);
                }
        // pairs of k-blocks: lane L's uint2 of k-blocks 2j and 2j + 1 side by side
        vt[(((int64_t)rg * (KB1e >> 1) + (kb >> 1)) * 32 + lane) * 2 + (kb & 1)] = make_uint2(w[0], w[1]);
    }
}

// Contraction-2 tiles: rows are the N outputs, k runs over the latent indices
// of both paths (path p owns k in [p*r32, p*r32 + r32)).  Bit = U_sign[n][j] < 0.
__global__ void build_utiles_kernel(uint2 *__restrict__ ut, int RG2, int KB2e, int r, int r32, int N,
                                    int npaths, const uint32_t *__restrict__ U0,
                                    const uint32_t *__restrict__ U1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RG2 * KB2e * 32;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t u = idx >> 5;
        const int kb = (int)(u % KB2e);
        const int rg = (int)(u / KB2e);
        const int g = lane >> 2, t = lane & 3;
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int n = rg * kRowsPerGroup + 16 * (i & 3) + g + 8 * (i >> 2);
                    const int jj = kb * kKPerBlock + 4 * t + b + 16 * q;
                    const int p = jj / r32;
                    const int j = jj - p * r32;
                    if (p < npaths && j < r && n < N)
                        w[q] |= canon_bit(p ? U1 : U0, wpr, n, j) << (8 * b + i);
                }
        ut[(((int64_t)rg * (KB2e >> 1) + (kb >> 1)) * 32 + lane) * 2 + (kb & 1)] = make_uint2(w[0], w[1]);
    }
}

// dst[p][0..npad) = src_p[0..n) followed by zeros.
__global__ void pad_copy_kernel(uint16_t *__restrict__ dst, const uint16_t *__restrict__ s0,
                                const uint16_t *__restrict__ s1, int npaths, int n, int npad)
{
    const int64_t total = (int64_t)npaths * npad;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int p = (int)(idx / npad);
        const int i = (int)(idx - (int64_t)p * npad);
        dst[idx] = (i < n) ? (p ? s1 : s0)[i] : (uint16_t)0;
    }
}

// Row scales of contraction 2 in fragment order: for row group rg, path p and
// lane row g, the eight values h_p[64 rg + 16 rb + g + 8 hf] (rb < 4, hf < 2)
// are contiguous, [rg][p][g][rb][hf]; zero for an absent path or row >= N.
__global__ void build_hq_kernel(uint16_t *__restrict__ hq, int RG2, int N, int npaths,
                                const uint16_t *__restrict__ h0, const uint16_t *__restrict__ h1)
{
    const int64_t total = (int64_t)RG2 * 128;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int w = (int)(idx & 127);
        const int rg = (int)(idx >> 7);
        const int p = w >> 6, g = (w >> 3) & 7, rb = (w >> 1) & 3, hf = w & 1;
        const int row = rg * kRowsPerGroup + 16 * rb + g + 8 * hf;
        hq[idx] = (p < npaths && row < N) ? (p ? h1 : h0)[row] : (uint16_t)0;
    }
}

static AttrCache g_attr_cache;

cudaError_t ensure_dyn_smem(const void *fn, size_t bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int r = g_attr_cache.ensure(dev, fn, (long)bytes, [&](long b) {
        return (int)cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b);
    });
    return (cudaError_t)r;
}

cudaError_t sm_count_of_current(int *sms)
{
    static std::mutex mu;
    static std::map<int, int> counts;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = counts.find(dev);
    if (it == counts.end()) {
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        it = counts.emplace(dev, n).first;
    }
    *sms = it->second;
    return cudaSuccess;
}

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

static int grid_for(int64_t work, int threads)
{
    int64_t b = (work + threads - 1) / threads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(b, 148 * 32));
}

// ---------------------------------------------------------------- plans

void plan_free(Plan &P)
{
    prefill_free(P.pf);
    if (P.dev) cudaFree(P.dev);
    if (P.p1) cudaFree(P.p1);
    if (P.p2) cudaFree(P.p2);
    if (P.sg1) cudaFree(P.sg1);
    if (P.sg2) cudaFree(P.sg2);
    if (P.bnd1) cudaFree(P.bnd1);
    if (P.bnd2) cudaFree(P.bnd2);
    if (P.cls1) cudaFree(P.cls1);
    if (P.cls2) cudaFree(P.cls2);
    if (P.scratch) cudaFree(P.scratch);
    P = Plan();
}

cudaError_t plan_build(Plan &P, const lb_layer *const *layers, int n, cudaStream_t s)
{
    P.n = n;
    P.layers.assign(layers, layers + n);
    P.host.resize(n);
    // scratch layout
    std::vector<size_t> off(n);
    size_t total = 0;
    for (int i = 0; i < n; ++i) {
        const LayerDev &d = layers[i]->d;
        off[i] = total;
        total += align256(acc_doubles(d.R1) * sizeof(double));
        total += align256((size_t)kMaxNT * d.KB2 * 32 * sizeof(uint2));
        total += align256((size_t)2 * 16 * sizeof(int2));
        total += align256(sizeof(unsigned));
        total += align256((size_t)d.KB1e * 32 * sizeof(uint2));
        total += align256((size_t)d.nkc * 4 * sizeof(int));
    }
    total += 256;   // error code
    cudaError_t e = cudaMalloc(&P.scratch, std::max<size_t>(total, 256));
    if (e != cudaSuccess) return e;
    P.scratch_bytes = total;
    e = cudaMemsetAsync(P.scratch, 0, total, s);
    if (e != cudaSuccess) return e;
    char *base = (char *)P.scratch;
    for (int i = 0; i < n; ++i) {
        LayerDev d = layers[i]->d;
        char *c = base + off[i];
        d.acc = (double *)c;       c += align256(acc_doubles(d.R1) * sizeof(double));
        d.zfrag = (uint2 *)c;      c += align256((size_t)kMaxNT * d.KB2 * 32 * sizeof(uint2));
        d.zmeta = (int2 *)c;       c += align256((size_t)2 * 16 * sizeof(int2));
        d.xfrag = (uint2 *)c;      c += align256((size_t)d.KB1e * 32 * sizeof(uint2));
        d.xmeta = (int *)c;
        P.host[i] = d;
    }
    P.err = (int *)(base + total - 256);
    // work items, layer-major; one IO batch per kIoBatch layers
    std::vector<P1Item> p1;
    std::vector<P2Item> p2;
    for (int i = 0; i < n; ++i) {
        if (i % kIoBatch == 0) {
            P.p1_start.push_back((int)p1.size());
            P.p2_start.push_back((int)p2.size());
        }
        const LayerDev &d = P.host[i];
        for (int kc = 0; kc < d.nkc; ++kc) p1.push_back({i, kc});
        for (int rg = 0; rg < d.RG2; rg += kP2ItemGroups)
            p2.push_back({i, rg, std::min(rg + kP2ItemGroups, d.RG2), 0});
    }
    P.p1_start.push_back((int)p1.size());
    P.p2_start.push_back((int)p2.size());
    // Within a launch, hand out the largest items first: static round-robin over a
    // largest-first list keeps the tail of the grid short.
    auto w1 = [&](const P1Item &a) {
        const LayerDev &d = P.host[a.layer];
        return (long long)d.RG1 * std::min(kP1ChunkKB, d.KB1 - a.kc * kP1ChunkKB);
    };
    auto w2 = [&](const P2Item &a) { return (long long)(a.rg1 - a.rg0) * P.host[a.layer].KB2; };
    for (size_t b = 0; b + 1 < P.p1_start.size(); ++b) {
        std::stable_sort(p1.begin() + P.p1_start[b], p1.begin() + P.p1_start[b + 1],
                         [&](const P1Item &a, const P1Item &c) { return w1(a) > w1(c); });
        std::stable_sort(p2.begin() + P.p2_start[b], p2.begin() + P.p2_start[b + 1],
                         [&](const P2Item &a, const P2Item &c) { return w2(a) > w2(c); });
    }
    P.n_p1 = (int)p1.size();
    P.n_p2 = (int)p2.size();

    // Segments of the one/two-row streaming kernels, per IO batch.  A unit takes H = ceil(P / 2) steps (P pairs
    // of k-blocks, two per step); the kernels have unrolled paths for some H (the static classes) and a generic
    // loop for the rest.  The batch's units are grouped by class (layer order within a class), every class gets
    // a share of the #SM * kLdgWarps warps in proportion to its estimated cost, and each class's units are split
    // into contiguous ranges of equal cost, one per warp, cut into segments (runs of one layer; in contraction 1
    // of one chunk).  Range r goes to warp r / #SM of CTA r % #SM, so each SM holds ranges of every class.
    int sms = 148, dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    P.kb2max = 0;
    P.rmax = 0;
    for (int i = 0; i < n; ++i) {
        P.kb2max = std::max(P.kb2max, P.host[i].KB2);
        P.rmax = std::max(P.rmax, P.host[i].r);
    }
    P.stream_grid = sms;
    const int nwarps = sms * kLdgWarps;
    std::vector<Seg1> sg1;
    std::vector<Seg2> sg2;
    std::vector<int> bnd1, bnd2, cls1, cls2;
    const int nb = (int)P.p1_start.size() - 1;
    // a unit: layer, linear index within the layer, pairs, cost (k-blocks plus the epilogue; the generic loop
    // runs slower per k-block)
    struct Unit { int layer, ul, P; double cost; };
    auto class1 = [](int pairs) { const int H = (pairs + 1) / 2; return (H == 6 || H == 8) ? H : 0; };
    auto class2 = [](int pairs) {
        const int H = (pairs + 1) / 2;
        return ((H >= 1 && H <= 6) || H == 9 || H == 13) ? H : 0;
    };
    // a unit's k-blocks plus its epilogue and block bookkeeping, in k-block equivalents (fitted to per-warp times
    // on B200); the generic loop runs about a third slower
    auto unit_cost = [](int pairs, int cls) { return (2.0 * pairs + 16.0) * (cls ? 1.0 : 1.35); };
    // ranges[r] = (class, first unit, end unit) over `order` (unit indices grouped by class)
    auto partition = [&](const std::vector<Unit> &us, auto class_of, std::vector<int> &order,
                         std::vector<std::array<int, 3>> &ranges) {
        std::vector<int> classes;
        for (const Unit &x : us) {
            const int c = class_of(x.P);
            if (std::find(classes.begin(), classes.end(), c) == classes.end()) classes.push_back(c);
        }
        std::sort(classes.begin(), classes.end());
        std::vector<double> cost(classes.size(), 0.0);
        order.clear();
        std::vector<size_t> cstart;
        for (size_t ci = 0; ci < classes.size(); ++ci) {
            cstart.push_back(order.size());
            for (size_t u = 0; u < us.size(); ++u)
                if (class_of(us[u].P) == classes[ci]) {
                    order.push_back((int)u);
                    cost[ci] += us[u].cost;
                }
        }
        cstart.push_back(order.size());
        double total = 0.0;
        for (double c : cost) total += c;
        // warps per class: at least one each, the rest by largest remainder
        std::vector<int> nw(classes.size(), 1);
        int left = nwarps - (int)classes.size();
        std::vector<double> want(classes.size());
        for (size_t ci = 0; ci < classes.size(); ++ci) want[ci] = total > 0 ? cost[ci] / total * left : 0.0;
        for (size_t ci = 0; ci < classes.size(); ++ci) {
            nw[ci] += (int)want[ci];
            left -= (int)want[ci];
        }
        while (left > 0) {
            size_t best = 0;
            for (size_t ci = 1; ci < classes.size(); ++ci)
                if (want[ci] - (int)want[ci] > want[best] - (int)want[best]) best = ci;
            ++nw[best];
            want[best] = (int)want[best];     // its remainder is used up
            --left;
        }
        ranges.clear();
        for (size_t ci = 0; ci < classes.size(); ++ci) {
            const size_t a0 = cstart[ci], a1 = cstart[ci + 1];
            size_t u = a0;
            double acc = 0.0;
            for (int w = 0; w < nw[ci]; ++w) {
                const double target = cost[ci] * (w + 1) / nw[ci];
                const size_t first = u;
                while (u < a1 && (w + 1 == nw[ci] || acc + 0.5 * us[order[u]].cost < target)) acc += us[order[u++]].cost;
                ranges.push_back({classes[ci], (int)first, (int)u});
            }
        }
    };
    for (int b = 0; b < nb; ++b) {
        const int l0 = b * kIoBatch, l1 = std::min(n, l0 + kIoBatch);
        std::vector<Unit> us1, us2;
        for (int i = l0; i < l1; ++i) {
            const LayerDev &d = P.host[i];
            for (int kc = 0; kc < d.nkc; ++kc) {
                const int pairs = (std::min(kP1ChunkKB, d.KB1 - kc * kP1ChunkKB) + 1) / 2;
                for (int rg = 0; rg < d.RG1; ++rg)
                    us1.push_back({i, kc * d.RG1 + rg, pairs, unit_cost(pairs, class1(pairs))});
            }
            for (int rg = 0; rg < d.RG2; ++rg) us2.push_back({i, rg, d.KB2e / 2, unit_cost(d.KB2e / 2, class2(d.KB2e / 2))});
        }
        std::vector<int> o1, o2;
        std::vector<std::array<int, 3>> r1, r2;
        partition(us1, class1, o1, r1);
        partition(us2, class2, o2, r2);
        const size_t first1 = bnd1.size(), first2 = bnd2.size();
        bnd1.resize(first1 + nwarps + 1);
        bnd2.resize(first2 + nwarps + 1);
        const size_t fc1 = cls1.size(), fc2 = cls2.size();
        cls1.resize(fc1 + nwarps, 0);
        cls2.resize(fc2 + nwarps, 0);
        std::vector<std::vector<Seg1>> per1(nwarps);
        std::vector<std::vector<Seg2>> per2(nwarps);
        for (int r = 0; r < nwarps; ++r) {
            const int w = (r % sms) * kLdgWarps + r / sms;
            cls1[fc1 + w] = r1[r][0];
            for (int a = r1[r][1]; a < r1[r][2];) {
                // units of one layer and one chunk: ul = kc * RG1 + rg (consecutive in `order` within a class)
                const Unit &f = us1[o1[a]];
                const LayerDev &d = P.host[f.layer];
                const int kc = f.ul / d.RG1, rg0 = f.ul - kc * d.RG1;
                int e2 = a + 1;
                while (e2 < r1[r][2] && us1[o1[e2]].layer == f.layer && us1[o1[e2]].ul == f.ul + (e2 - a) &&
                       us1[o1[e2]].ul / d.RG1 == kc)
                    ++e2;
                per1[w].push_back({reinterpret_cast<const uint4 *>(d.vt) +
                                       ((size_t)rg0 * (d.KB1e / 2) + (size_t)kc * (kP1ChunkKB / 2)) * 32,
                                   f.layer, kc, rg0, e2 - a, f.P, d.KB1e / 2 * 32});
                a = e2;
            }
            cls2[fc2 + w] = r2[r][0];
            for (int a = r2[r][1]; a < r2[r][2];) {
                const Unit &f = us2[o2[a]];
                const LayerDev &d = P.host[f.layer];
                int e2 = a + 1;
                while (e2 < r2[r][2] && us2[o2[e2]].layer == f.layer && us2[o2[e2]].ul == f.ul + (e2 - a)) ++e2;
                per2[w].push_back({reinterpret_cast<const uint4 *>(d.ut) + (size_t)f.ul * (d.KB2e / 2) * 32,
                                   d.hq + (size_t)f.ul * 16, f.layer, f.ul, e2 - a, d.KB2e / 2});
                a = e2;
            }
        }
        for (int w = 0; w < nwarps; ++w) {
            bnd1[first1 + w] = (int)sg1.size();
            sg1.insert(sg1.end(), per1[w].begin(), per1[w].end());
            bnd2[first2 + w] = (int)sg2.size();
            sg2.insert(sg2.end(), per2[w].begin(), per2[w].end());
        }
        bnd1[first1 + nwarps] = (int)sg1.size();
        bnd2[first2 + nwarps] = (int)sg2.size();
    }
    if ((e = cudaMalloc(&P.sg1, sizeof(Seg1) * std::max<size_t>(1, sg1.size()))) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.sg2, sizeof(Seg2) * std::max<size_t>(1, sg2.size()))) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.bnd1, sizeof(int) * bnd1.size())) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.bnd2, sizeof(int) * bnd2.size())) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.cls1, sizeof(int) * std::max<size_t>(1, cls1.size()))) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.cls2, sizeof(int) * std::max<size_t>(1, cls2.size()))) != cudaSuccess) return e;
    if (!sg1.empty() && (e = cudaMemcpy(P.sg1, sg1.data(), sizeof(Seg1) * sg1.size(), cudaMemcpyHostToDevice)) !=
                            cudaSuccess)
        return e;
    if (!sg2.empty() && (e = cudaMemcpy(P.sg2, sg2.data(), sizeof(Seg2) * sg2.size(), cudaMemcpyHostToDevice)) !=
                            cudaSuccess)
        return e;
    if ((e = cudaMemcpy(P.bnd1, bnd1.data(), sizeof(int) * bnd1.size(), cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    if ((e = cudaMemcpy(P.bnd2, bnd2.data(), sizeof(int) * bnd2.size(), cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    if (!cls1.empty() && (e = cudaMemcpy(P.cls1, cls1.data(), sizeof(int) * cls1.size(), cudaMemcpyHostToDevice)) !=
                             cudaSuccess)
        return e;
    if (!cls2.empty() && (e = cudaMemcpy(P.cls2, cls2.data(), sizeof(int) * cls2.size(), cudaMemcpyHostToDevice)) !=
                             cudaSuccess)
        return e;

    if ((e = cudaMalloc(&P.dev, sizeof(LayerDev) * n)) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.p1, sizeof(P1Item) * std::max(1, P.n_p1))) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.p2, sizeof(P2Item) * std::max(1, P.n_p2))) != cudaSuccess) return e;
    // synchronous copies from pageable memory: the host vectors die with this call
    if ((e = cudaMemcpy(P.dev, P.host.data(), sizeof(LayerDev) * n, cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    if ((e = cudaMemcpy(P.p1, p1.data(), sizeof(P1Item) * P.n_p1, cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    if ((e = cudaMemcpy(P.p2, p2.data(), sizeof(P2Item) * P.n_p2, cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    return cudaSuccess;
}

}  // namespace lb

using namespace lb;

// M <= LB_DECODE_MAX_M: fused decode kernels.  Larger M: tensor-core kernels;
// shapes those cannot take (K not a multiple of 8) run as 16-row decode blocks.
static lb_status forward_any(const Plan &P, const uint16_t *const *xs, float *const *ys, int M, cudaStream_t s,
                             int *launches)
{
    if (M > kMaxDecodeM) {
        lb_status st = prefill_forward(P, P.layers.data(), xs, ys, M, s, launches);
        if (st != LB_ERR_UNSUPPORTED) return st;
    }
    return decode_forward(P, xs, ys, M, s, launches);
}

extern "C" {

lb_status lb_layer_create(lb_layer **out, int N, int K, int r, int npaths, const uint32_t *const *U,
                          const uint32_t *const *V, const uint16_t *const *h,
                          const uint16_t *const *g, const uint16_t *const *l, void *stream)
{
    set_launch_count(0);
    if (!out) return LB_ERR_INVALID_ARG;
    *out = nullptr;
    if (N < 1 || K < 1 || r < 1 || r > LB_MAX_RANK) return LB_ERR_INVALID_ARG;
    if (npaths != 1 && npaths != 2) return LB_ERR_UNSUPPORTED;
    if (!U || !V || !h || !g || !l) return LB_ERR_INVALID_ARG;
    for (int p = 0; p < npaths; ++p)
        if (!U[p] || !V[p] || !h[p] || !g[p] || !l[p]) return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;

    lb_layer *L = new (std::nothrow) lb_layer();
    if (!L) return LB_ERR_OOM;
    LayerDev &d = L->d;
    std::memset(&d, 0, sizeof(d));
    d.N = N; d.K = K; d.r = r; d.npaths = npaths;
    d.r16 = round_up(r, 16);
    d.r32 = round_up(r, 32);
    d.R1 = round_up(npaths * d.r16, kRowsPerGroup);
    d.RG1 = d.R1 / kRowsPerGroup;
    d.K32 = round_up(K, kKPerBlock);
    d.KB1 = d.K32 / kKPerBlock;
    d.N64 = round_up(N, kRowsPerGroup);
    d.RG2 = d.N64 / kRowsPerGroup;
    d.KB2 = npaths * d.r32 / kKPerBlock;
    d.nkc = ceil_div(d.KB1, kP1ChunkKB);
    d.KB1e = round_up(d.KB1, 2);
    d.KB2e = round_up(d.KB2, 2);

    // one pair of k-blocks (512 bytes) of padding after each tile array: the streaming kernels may read the pair
    // after a unit whose pair count is odd (with a zero B fragment)
    const size_t b_vt = align256((size_t)d.RG1 * d.KB1e * 32 * sizeof(uint2) + 512);
    const size_t b_ut = align256((size_t)d.RG2 * d.KB2e * 32 * sizeof(uint2) + 512);
    const size_t b_g = align256((size_t)npaths * d.K32 * 2);
    const size_t b_h = align256((size_t)npaths * d.N64 * 2);
    const size_t b_l = align256((size_t)npaths * d.r16 * 2);
    const size_t b_hq = align256((size_t)d.RG2 * 256);
    const size_t b_pf = prefill_weight_bytes(d);
    L->weight_bytes = b_vt + b_ut + b_g + b_h + b_l + b_hq + b_pf;
    cudaError_t e = cudaMalloc(&L->weights, L->weight_bytes);
    if (e != cudaSuccess) {
        delete L;
        return status_from(e);
    }
    char *c = (char *)L->weights;
    d.vt = (const uint2 *)c;   c += b_vt;
    d.ut = (const uint2 *)c;   c += b_ut;
    d.g = (const __half *)c;   c += b_g;
    d.h = (const __half *)c;   c += b_h;
    d.l = (const __half *)c;   c += b_l;
    d.hq = (const uint4 *)c;   c += b_hq;
    L->pf.b1 = (uint32_t *)c;  // prefill layouts are carved from here

    const int T = 256;
    const uint32_t *V1 = npaths > 1 ? V[1] : V[0];
    const uint32_t *U1 = npaths > 1 ? U[1] : U[0];
    int launches = 0;
    build_vtiles_kernel<<<grid_for((int64_t)d.RG1 * d.KB1e * 32, T), T, 0, s>>>(
        (uint2 *)d.vt, d.RG1, d.KB1e, r, d.r16, K, npaths, V[0], V1);
    build_utiles_kernel<<<grid_for((int64_t)d.RG2 * d.KB2e * 32, T), T, 0, s>>>(
        (uint2 *)d.ut, d.RG2, d.KB2e, r, d.r32, N, npaths, U[0], U1);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.K32, T), T, 0, s>>>(
        (uint16_t *)d.g, g[0], npaths > 1 ? g[1] : g[0], npaths, K, d.K32);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.N64, T), T, 0, s>>>(
        (uint16_t *)d.h, h[0], npaths > 1 ? h[1] : h[0], npaths, N, d.N64);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.r16, T), T, 0, s>>>(
        (uint16_t *)d.l, l[0], npaths > 1 ? l[1] : l[0], npaths, r, d.r16);
    build_hq_kernel<<<grid_for((int64_t)d.RG2 * 128, T), T, 0, s>>>((uint16_t *)d.hq, d.RG2, N, npaths, h[0],
                                                                     npaths > 1 ? h[1] : h[0]);
    launches = 6;
    e = cudaGetLastError();
    if (e == cudaSuccess) {
        e = prefill_build_weights(L->pf, d, U, V, h, g, l, s);
        launches += 5;
    }
    if (e == cudaSuccess) {
        lb_stack *S = new (std::nothrow) lb_stack();
        if (!S) {
            e = cudaErrorMemoryAllocation;
        } else {
            S->layers.push_back(L);
            const lb_layer *one = L;
            e = plan_build(S->plan, &one, 1, s);
            L->self = S;
        }
    }
    if (e != cudaSuccess) {
        lb_layer_destroy(L);
        return status_from(e);
    }
    set_launch_count(launches);
    *out = L;
    return LB_OK;
}

void lb_layer_destroy(lb_layer *L)
{
    if (!L) return;
    cudaDeviceSynchronize();
    if (L->self) {
        plan_free(L->self->plan);
        delete L->self;
    }
    if (L->weights) cudaFree(L->weights);
    delete L;
}

lb_status lb_layer_shape(const lb_layer *L, int *N, int *K, int *r, int *npaths)
{
    if (!L) return LB_ERR_INVALID_ARG;
    if (N) *N = L->d.N;
    if (K) *K = L->d.K;
    if (r) *r = L->d.r;
    if (npaths) *npaths = L->d.npaths;
    return LB_OK;
}

double lb_layer_bpw(const lb_layer *L)
{
    if (!L) return 0.0;
    const double N = L->d.N, K = L->d.K, r = L->d.r;
    return L->d.npaths * (r * (N + K) + 16.0 * (N + K + r)) / (N * K);
}

size_t lb_layer_device_bytes(const lb_layer *L)
{
    if (!L) return 0;
    size_t b = L->weight_bytes;
    if (L->self) b += L->self->plan.scratch_bytes;
    return b;
}

lb_status lb_linear_forward(const uint16_t *x, int M, const lb_layer *L, float *y, void *stream)
{
    set_launch_count(0);
    if (!L || M < 0) return LB_ERR_INVALID_ARG;
    if (M == 0) return LB_OK;
    if (!x || !y || ((uintptr_t)x & 15) || ((uintptr_t)y & 15)) return LB_ERR_INVALID_ARG;
    const uint16_t *xs[1] = {x};
    float *ys[1] = {y};
    int launches = 0;
    lb_status st = forward_any(L->self->plan, xs, ys, M, (cudaStream_t)stream, &launches);
    set_launch_count(launches);
    return st;
}

lb_status lb_stack_create(lb_stack **out, const lb_layer *const *layers, int n, void *stream)
{
    set_launch_count(0);
    if (!out) return LB_ERR_INVALID_ARG;
    *out = nullptr;
    if (!layers || n < 1 || n > LB_STACK_MAX_LAYERS) return LB_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!layers[i]) return LB_ERR_INVALID_ARG;
    lb_stack *S = new (std::nothrow) lb_stack();
    if (!S) return LB_ERR_OOM;
    S->layers.assign(layers, layers + n);
    cudaError_t e = plan_build(S->plan, layers, n, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        plan_free(S->plan);
        delete S;
        return status_from(e);
    }
    *out = S;
    return LB_OK;
}

void lb_stack_destroy(lb_stack *S)
{
    if (!S) return;
    cudaDeviceSynchronize();
    plan_free(S->plan);
    delete S;
}

lb_status lb_stack_forward(lb_stack *S, const uint16_t *const *xs, float *const *ys, int M, void *stream)
{
    set_launch_count(0);
    if (!S || M < 0) return LB_ERR_INVALID_ARG;
    if (M == 0) return LB_OK;
    if (!xs || !ys) return LB_ERR_INVALID_ARG;
    for (int i = 0; i < S->plan.n; ++i)
        if (!xs[i] || !ys[i] || ((uintptr_t)xs[i] & 15) || ((uintptr_t)ys[i] & 15))
            return LB_ERR_INVALID_ARG;
    int launches = 0;
    lb_status st = forward_any(S->plan, xs, ys, M, (cudaStream_t)stream, &launches);
    set_launch_count(launches);
    return st;
}

}  // extern "C"
