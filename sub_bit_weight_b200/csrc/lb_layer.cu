// Layer objects, their private weight layouts, execution plans and stacks.
//
// A layer is built from the canonical packed signs (one bit per sign, sign(0)
// = +1) and binary16 scales of its two paths (LittleBit notes page,
// "Multi-scale compensation" and "Residual compensation").  It re-tiles the
// signs into the layouts its kernels stream (see lb_internal.cuh) and keeps
// the scales zero-padded, so padded rank slots and rows contribute nothing.

#include <algorithm>
#include <cstring>
#include <new>

#include "lb_prefill.cuh"

namespace lb {

__device__ __forceinline__ uint32_t canon_bit(const uint32_t *P, int wpr, int64_t row, int col)
{
    return (__ldg(P + row * wpr + (col >> 5)) >> (col & 31)) & 1u;
}

// Contraction-1 tiles: rows are latent indices of both paths (path p owns
// rows [p*r16, p*r16 + r16)), k runs over the K inputs.  Bit = V_sign[k][j] < 0.
__global__ void build_vtiles_kernel(uint2 *__restrict__ vt, int RG1, int KB1, int r, int r16, int K,
                                    int npaths, const uint32_t *__restrict__ V0,
                                    const uint32_t *__restrict__ V1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RG1 * KB1 * 32;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t u = idx >> 5;
        const int kb = (int)(u % KB1);
        const int rg = (int)(u / KB1);
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
        vt[idx] = make_uint2(w[0], w[1]);
    }
}

// Contraction-2 tiles: rows are the N outputs, k runs over the latent indices
// of both paths (path p owns k in [p*r32, p*r32 + r32)).  Bit = U_sign[n][j] < 0.
__global__ void build_utiles_kernel(uint2 *__restrict__ ut, int RG2, int KB2, int r, int r32, int N,
                                    int npaths, const uint32_t *__restrict__ U0,
                                    const uint32_t *__restrict__ U1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RG2 * KB2 * 32;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(idx & 31);
        const int64_t u = idx >> 5;
        const int kb = (int)(u % KB2);
        const int rg = (int)(u / KB2);
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
        ut[idx] = make_uint2(w[0], w[1]);
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
    if (P.u1) cudaFree(P.u1);
    if (P.u2) cudaFree(P.u2);
    for (int mm = 0; mm < 2; ++mm) {
        if (P.wr1[mm]) cudaFree(P.wr1[mm]);
        if (P.wr2[mm]) cudaFree(P.wr2[mm]);
    }
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
        total += align256((size_t)d.KB1 * 32 * sizeof(uint2));
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
        d.xfrag = (uint2 *)c;      c += align256((size_t)d.KB1 * 32 * sizeof(uint2));
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

    // One/two-row streaming units in layer order, and per batch an equal split
    // of their estimated cost over pair_warps warps (warp w streams units
    // [wr[w], wr[w + 1]) of its batch).
    int sms = 148, dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    P.kb2max = 0;
    P.rmax = 0;
    for (int i = 0; i < n; ++i) {
        P.kb2max = std::max(P.kb2max, P.host[i].KB2);
        P.rmax = std::max(P.rmax, P.host[i].r);
    }
    std::vector<PairUnit1> u1;
    std::vector<PairUnit2> u2;
    std::vector<int> wr1[2], wr2[2];
    const int nb = (int)P.p1_start.size() - 1;
    // contraction 1: cost in issued instructions per warp (MMA k-blocks, ring stages, per-unit epilogue)
    auto stages = [](int nkb) { return (double)((nkb + kPairStageKB - 1) / kPairStageKB); };
    auto cost1 = [&](const PairUnit1 &u) { return 22.0 * u.nkb + 40.0 * stages(u.nkb) + 60.0; };
    // contraction 2, in k-block equivalents (fitted to per-warp times on B200): a k-block, 8.5 per row group
    // (fold, h, stores), 15 where a layer starts (its zl fragments are waited for)
    auto cost2 = [&](const PairUnit2 &u) { return (double)u.kb2 + 8.5 + (u.rg == 0 ? 15.0 : 0.0); };
    for (int b = 0; b < nb; ++b) {
        const int l0 = b * kIoBatch, l1 = std::min(n, l0 + kIoBatch);
        const size_t s1 = u1.size(), s2 = u2.size();
        for (int i = l0; i < l1; ++i) {
            const LayerDev &d = P.host[i];
            for (int kc = 0; kc < d.nkc; ++kc) {
                const int nkb = std::min(kP1ChunkKB, d.KB1 - kc * kP1ChunkKB);
                for (int rg = 0; rg < d.RG1; ++rg)
                    u1.push_back({d.vt + ((size_t)rg * d.KB1 + (size_t)kc * kP1ChunkKB) * 32, i, kc, rg, nkb});
            }
            for (int rg = 0; rg < d.RG2; ++rg) u2.push_back({d.ut + (size_t)rg * d.KB2 * 32, i, rg, d.KB2, 0});
        }
        // per row count: an equal split of the estimated cost over all warps of one CTA per SM
        for (int mm = 0; mm < 2; ++mm) {
            const int W1 = sms * pair_warps_per_cta(mm + 1);
            const int W2 = sms * pair2_warps_per_cta(mm + 1, std::min(P.kb2max, kPairMaxKB2));
            P.pair_warps[mm] = W1;
            P.pair_warps2[mm] = W2;
            auto split = [&](std::vector<int> &wr, size_t first, size_t last, int W, auto cost_of) {
                double total_c = 0.0;
                for (size_t u = first; u < last; ++u) total_c += cost_of(u);
                size_t u = first;
                double acc = 0.0;
                for (int w = 0; w <= W; ++w) {
                    const double target = total_c * w / W;
                    while (u < last && acc + 0.5 * cost_of(u) < target) acc += cost_of(u++);
                    wr.push_back((int)(w == W ? last : u));
                }
            };
            split(wr1[mm], s1, u1.size(), W1, [&](size_t u) { return cost1(u1[u]); });
            split(wr2[mm], s2, u2.size(), W2, [&](size_t u) { return cost2(u2[u]); });
        }
    }
    if ((e = cudaMalloc(&P.u1, sizeof(PairUnit1) * std::max<size_t>(1, u1.size()))) != cudaSuccess) return e;
    if ((e = cudaMalloc(&P.u2, sizeof(PairUnit2) * std::max<size_t>(1, u2.size()))) != cudaSuccess) return e;
    if (!u1.empty() && (e = cudaMemcpy(P.u1, u1.data(), sizeof(PairUnit1) * u1.size(), cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    if (!u2.empty() && (e = cudaMemcpy(P.u2, u2.data(), sizeof(PairUnit2) * u2.size(), cudaMemcpyHostToDevice)) != cudaSuccess)
        return e;
    for (int mm = 0; mm < 2; ++mm) {
        if ((e = cudaMalloc(&P.wr1[mm], sizeof(int) * std::max<size_t>(1, wr1[mm].size()))) != cudaSuccess) return e;
        if ((e = cudaMalloc(&P.wr2[mm], sizeof(int) * std::max<size_t>(1, wr2[mm].size()))) != cudaSuccess) return e;
        if ((e = cudaMemcpy(P.wr1[mm], wr1[mm].data(), sizeof(int) * wr1[mm].size(), cudaMemcpyHostToDevice)) !=
            cudaSuccess)
            return e;
        if ((e = cudaMemcpy(P.wr2[mm], wr2[mm].data(), sizeof(int) * wr2[mm].size(), cudaMemcpyHostToDevice)) !=
            cudaSuccess)
            return e;
    }

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

    const size_t b_vt = align256((size_t)d.RG1 * d.KB1 * 32 * sizeof(uint2));
    const size_t b_ut = align256((size_t)d.RG2 * d.KB2 * 32 * sizeof(uint2));
    const size_t b_g = align256((size_t)npaths * d.K32 * 2);
    const size_t b_h = align256((size_t)npaths * d.N64 * 2);
    const size_t b_l = align256((size_t)npaths * d.r16 * 2);
    const size_t b_pf = prefill_weight_bytes(d);
    L->weight_bytes = b_vt + b_ut + b_g + b_h + b_l + b_pf;
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
    L->pf.b1 = (uint32_t *)c;  // prefill layouts are carved from here

    const int T = 256;
    const uint32_t *V1 = npaths > 1 ? V[1] : V[0];
    const uint32_t *U1 = npaths > 1 ? U[1] : U[0];
    int launches = 0;
    build_vtiles_kernel<<<grid_for((int64_t)d.RG1 * d.KB1 * 32, T), T, 0, s>>>(
        (uint2 *)d.vt, d.RG1, d.KB1, r, d.r16, K, npaths, V[0], V1);
    build_utiles_kernel<<<grid_for((int64_t)d.RG2 * d.KB2 * 32, T), T, 0, s>>>(
        (uint2 *)d.ut, d.RG2, d.KB2, r, d.r32, N, npaths, U[0], U1);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.K32, T), T, 0, s>>>(
        (uint16_t *)d.g, g[0], npaths > 1 ? g[1] : g[0], npaths, K, d.K32);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.N64, T), T, 0, s>>>(
        (uint16_t *)d.h, h[0], npaths > 1 ? h[1] : h[0], npaths, N, d.N64);
    pad_copy_kernel<<<grid_for((int64_t)npaths * d.r16, T), T, 0, s>>>(
        (uint16_t *)d.l, l[0], npaths > 1 ? l[1] : l[0], npaths, r, d.r16);
    launches = 5;
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
