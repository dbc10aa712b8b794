// k_router.cuh -- DeepSeek-V3-style sigmoid router with group-limited top-k.
//
// README "JustVugg/colibri", section "已实现的功能": a DeepSeek-V3-like sigmoid
// router (noaux_tc, routed_scaling_factor).  The score-correction bias is
// used for selection only; groups are contiguous blocks of E/G experts scored
// by the sum of their two largest biased scores; the Gk best groups are kept;
// the k largest biased scores among their experts are chosen; weights are the
// unbiased scores renormalised over the choice and scaled by rsf.
//
// Two kernels: k_router_partial computes split-K partial dot products in
// double (tiles of 32 tokens x 64 experts, K split so that the grid fills the
// GPU even at one token); k_router_select sums the partials in split order,
// rounds the logit to f32 and selects, one warp per token.
#pragma once
#include "qrx_dev.cuh"

namespace qrx {

constexpr int RT_T = 32, RT_E = 64, RT_KC = 32;

template <bool XBF16>
__global__ void __launch_bounds__(256) k_router_partial(RouterArgs a, int kchunks_per_split)
{
    __shared__ double xs[RT_T][RT_KC + 1];
    __shared__ double wsm[RT_E][RT_KC + 1];
    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * RT_E, t0 = blockIdx.y * RT_T, ks = blockIdx.z;
    const int nchunks = a.H / RT_KC;
    const int c0 = ks * kchunks_per_split;
    const int c1 = min(nchunks, c0 + kchunks_per_split);
    const int tx = tid & 15, ty = tid >> 4;
    double acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

    for (int ch = c0; ch < c1; ++ch) {
        const int kb = ch * RT_KC;
        // x tile: 32 tokens x 32 k = 1024 values, 4 per thread
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = tid + 256 * q;
            const int tt = idx >> 5, kk = idx & 31;
            const int t = t0 + tt;
            double v = 0.0;
            if (t < a.T) {
                if constexpr (XBF16) {
                    v = (double)__bfloat162float(
                        reinterpret_cast<const __nv_bfloat16 *>(a.x)[(int64_t)t * a.H + kb + kk]);
                } else {
                    v = (double)reinterpret_cast<const float *>(a.x)[(int64_t)t * a.H + kb + kk];
                }
            }
            xs[tt][kk] = v;
        }
        // W tile: 64 experts x 32 k = 2048 values, 8 per thread
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int idx = tid + 256 * q;
            const int ee = idx >> 5, kk = idx & 31;
            const int e = e0 + ee;
            wsm[ee][kk] = e < a.E ? (double)a.Wr[(int64_t)e * a.H + kb + kk] : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < RT_KC; ++kk) {
            const double x0 = xs[ty][kk], x1 = xs[ty + 16][kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const double w = wsm[tx + 16 * j][kk];
                acc[0][j] = fma(x0, w, acc[0][j]);
                acc[1][j] = fma(x1, w, acc[1][j]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
            if (t < a.T && e < a.E) a.partial[((int64_t)ks * a.T + t) * a.E + e] = acc[i][j];
        }
}

// One warp per token.  Dynamic shared memory per warp: s[E], sc[E] (f32),
// gscore[G] (f32), kept[G] (int).
__global__ void __launch_bounds__(256) k_router_select(RouterArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + wid;
    const int E = a.E, G = a.G, gs = a.E / a.G;
    const size_t per_warp = (size_t)(2 * E + 2 * G) * 4;
    float *s_s = reinterpret_cast<float *>(smem_raw + per_warp * wid);
    float *sc_s = s_s + E;
    float *gsc = sc_s + E;
    int *kept = reinterpret_cast<int *>(gsc + G);
    if (t >= a.T) return;

    for (int e = lane; e < E; e += 32) {
        double acc = 0.0;
        for (int ks = 0; ks < a.KS; ++ks) acc += a.partial[((int64_t)ks * a.T + t) * E + e];
        const float lg = (float)acc;
        const float s = (float)(1.0 / (1.0 + exp(-(double)lg)));
        s_s[e] = s;
        sc_s[e] = __fadd_rn(s, a.bias[e]);
    }
    __syncwarp();
    for (int g = lane; g < G; g += 32) {
        float top1 = -INFINITY, top2 = -INFINITY;
        for (int e = g * gs; e < (g + 1) * gs; ++e) {
            const float v = sc_s[e];
            if (v > top1) { top2 = top1; top1 = v; }
            else if (v > top2) { top2 = v; }
        }
        gsc[g] = gs >= 2 ? __fadd_rn(top1, top2) : top1;
    }
    __syncwarp();
    for (int g = lane; g < G; g += 32) {
        const float v = gsc[g];
        int rank = 0;
        for (int h = 0; h < G; ++h) {
            const float u = gsc[h];
            rank += (u > v) || (u == v && h < g);
        }
        kept[g] = rank < a.Gk;
    }
    __syncwarp();
    uint32_t taken = 0;   // bit i: expert lane + 32 i taken
    for (int j = 0; j < a.k; ++j) {
        float best = -INFINITY;
        int be = 0x7fffffff;
        for (int i = 0; lane + 32 * i < E; ++i) {
            const int e = lane + 32 * i;
            if (!kept[e / gs] || (taken >> i & 1u)) continue;
            const float v = sc_s[e];
            if (be == 0x7fffffff || v > best) { best = v; be = e; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const bool better = (oe != 0x7fffffff) &&
                                (be == 0x7fffffff || ob > best || (ob == best && oe < be));
            if (better) { best = ob; be = oe; }
        }
        if (be == 0x7fffffff) {      // cannot happen for a validated configuration
            if (lane == 0) raise_status(DERR_BOUNDS);
            return;
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == 0) a.idx[(int64_t)t * a.k + j] = be;
    }
    __syncwarp();
    if (lane == 0) {
        double ssum = 0.0;
        for (int j = 0; j < a.k; ++j) ssum += (double)s_s[a.idx[(int64_t)t * a.k + j]];
        for (int j = 0; j < a.k; ++j) {
            const float s = s_s[a.idx[(int64_t)t * a.k + j]];
            a.w[(int64_t)t * a.k + j] = (float)((double)s / ssum * (double)a.rsf);
        }
    }
}

int router_ksplit(int T, int H, int E, int num_sms)
{
    const int nchunks = H / RT_KC;
    const int base = ((E + RT_E - 1) / RT_E) * ((T + RT_T - 1) / RT_T);
    int want = (2 * num_sms + base - 1) / base;
    if (want < 1) want = 1;
    int cps = nchunks / want;
    if (cps < 1) cps = 1;
    return (nchunks + cps - 1) / cps;
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t st)
{
    const int nchunks = a.H / RT_KC;
    const int cps = (nchunks + a.KS - 1) / a.KS;
    dim3 grid((a.E + RT_E - 1) / RT_E, (a.T + RT_T - 1) / RT_T, a.KS);
    if (a.x_bf16) k_router_partial<true><<<grid, 256, 0, st>>>(a, cps);
    else k_router_partial<false><<<grid, 256, 0, st>>>(a, cps);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)8 * (2 * a.E + 2 * a.G) * 4;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(k_router_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return err;
    }
    k_router_select<<<(a.T + 7) / 8, 256, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qrx
