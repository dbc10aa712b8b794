// k_router.cuh -- DeepSeek-V3-style sigmoid router with group-limited top-k.
//
// README "JustVugg/colibri", section "已实现的功能": a DeepSeek-V3-like sigmoid
// router (noaux_tc, routed_scaling_factor).  The score-correction bias is
// used for selection only; groups are contiguous blocks of E/G experts scored
// by the sum of their two largest biased scores; the Gk best groups are kept;
// the k largest biased scores among their experts are chosen; weights are the
// unbiased scores renormalised over the choice and scaled by rsf.
//
// Logits are summed in double and rounded to f32 once.  Few tokens
// (T <= 64): k_router_gemv, two experts per CTA, each expert's row split over
// four warps that keep their quarter of the row in registers and run every
// token over it.  More tokens: k_router_tile, 32-token x 64-expert tiles
// staged in shared memory.  Then k_router_select, one warp per token: sigmoid,
// bias, group scores, group choice, top-k and weights, and (when asked)
// adaptive expert top-p on the result (README, "快速开始": the --topp knob),
// which k_topp_prune also applies on its own to a router output in memory.
#pragma once
#include <algorithm>
#include "qrx_dev.cuh"
#include "k_permute.cuh"

namespace qrx {

constexpr int RT_T = 32, RT_E = 64, RT_KC = 32;

constexpr int RG_ROWS = 2;           // experts per CTA in k_router_gemv
constexpr int RG_TMAX = 64;          // tokens k_router_gemv can handle
constexpr int RG_TSPLIT = 4;         // tokens above which the split-K tile kernel is used (when given its scratch)

template <bool XBF16>
__device__ __forceinline__ float4 load_x4(const void *x, int64_t off)
{
    if constexpr (XBF16) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(
            reinterpret_cast<const __nv_bfloat16 *>(x) + off);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        return make_float4(a.x, a.y, b.x, b.y);
    } else {
        return *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + off);
    }
}

// Few tokens: warp (row r, quarter q) holds Wr[r][q*H/4 .. (q+1)*H/4) in
// registers (float4 per lane, at most RG_W4 of them) and dots every token's
// matching quarter of x with it in double.
constexpr int RG_W4 = 12;            // float4 per lane: H/16/32 <= 12 -> H <= 6144

template <bool XBF16>
__global__ void __launch_bounds__(256) k_router_gemv(RouterArgs a)
{
    __shared__ double part[RG_ROWS][4][RG_TMAX];
    pdl_trigger();                       // reads only inputs; waits before it exits
    if (blockIdx.x == 0 && a.zero)
        for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int rl = w >> 2, q = w & 3;
    const int e = blockIdx.x * RG_ROWS + rl;
    const int n4 = a.H / 16;                 // float4 per quarter
    const int64_t k0 = (int64_t)q * (a.H / 4);
    float4 wv[RG_W4];
#pragma unroll
    for (int j = 0; j < RG_W4; ++j) {
        const int i4 = lane + 32 * j;
        wv[j] = (e < a.E && i4 < n4)
                    ? *reinterpret_cast<const float4 *>(a.Wr + (int64_t)e * a.H + k0 + 4 * i4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int t = 0; t < a.T; ++t) {
        double acc = 0.0;
#pragma unroll
        for (int j = 0; j < RG_W4; ++j) {
            const int i4 = lane + 32 * j;
            if (i4 < n4) {
                const float4 xv = load_x4<XBF16>(a.x, (int64_t)t * a.H + k0 + 4 * i4);
                acc = fma((double)xv.x, (double)wv[j].x, acc);
                acc = fma((double)xv.y, (double)wv[j].y, acc);
                acc = fma((double)xv.z, (double)wv[j].z, acc);
                acc = fma((double)xv.w, (double)wv[j].w, acc);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) part[rl][q][t] = acc;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < RG_ROWS * a.T; i += blockDim.x) {
        const int r = i / a.T, t = i % a.T;
        const int ee = blockIdx.x * RG_ROWS + r;
        if (ee < a.E)
            a.logits[(int64_t)t * a.E + ee] =
                (float)(((part[r][0][t] + part[r][1][t]) + part[r][2][t]) + part[r][3][t]);
    }
    pdl_wait();
}

// Many tokens: 32-token x 64-expert tiles, K in chunks of 32 through shared memory.
template <bool XBF16>
__global__ void __launch_bounds__(256) k_router_tile(RouterArgs a)
{
    __shared__ double xs[RT_T][RT_KC + 1];
    __shared__ double wsm[RT_E][RT_KC + 1];
    pdl_trigger();                       // reads only inputs; waits before it exits
    if (blockIdx.x == 0 && blockIdx.y == 0 && a.zero)
        for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * RT_E, t0 = blockIdx.y * RT_T;
    const int c0 = 0, c1 = a.H / RT_KC;
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
            if (t < a.T && e < a.E) a.logits[(int64_t)t * a.E + e] = (float)acc[i][j];
        }
    pdl_wait();
}


// Many tokens, split over K: a CTA computes the f64 partial dots of 64
// tokens x 64 experts over one K slice (32-wide chunks of x and Wr staged in
// shared memory, 4 x 4 outputs per thread); the CTA that finishes a tile's
// last slice (a per-tile counter that it resets) adds the slices' partials in
// slice order and rounds each logit to f32 once.  Slices keep the grid near
// two CTAs per SM when there are few token tiles.
constexpr int RS_T = 64, RS_E = 64, RS_KC = 32;

template <bool XBF16>
__global__ void __launch_bounds__(256) k_router_split(RouterArgs a, int nslice, double *part, int *tilecnt)
{
    __shared__ double xs[RS_KC][RS_T + 1];
    __shared__ double wsm[RS_KC][RS_E + 1];
    __shared__ int last;
    pdl_trigger();                       // reads only inputs; waits before it exits
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && a.zero)
        for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0u;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int e0 = blockIdx.x * RS_E, t0 = blockIdx.y * RS_T, sl = blockIdx.z;
    const int kper = a.H / nslice, kb0 = sl * kper;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int kb = kb0; kb < kb0 + kper; kb += RS_KC) {
        // x: 64 tokens x 32 k, 8 per thread; Wr: 64 experts x 32 k, 8 per thread
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int idx = tid + 256 * q;
            const int rr = idx >> 5, kk = idx & 31;
            const int t = t0 + rr, e = e0 + rr;
            double xv = 0.0;
            if (t < a.T) {
                if constexpr (XBF16)
                    xv = (double)__bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(a.x)[(int64_t)t * a.H + kb + kk]);
                else
                    xv = (double)reinterpret_cast<const float *>(a.x)[(int64_t)t * a.H + kb + kk];
            }
            xs[kk][rr] = xv;
            wsm[kk][rr] = e < a.E ? (double)a.Wr[(int64_t)e * a.H + kb + kk] : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < RS_KC; ++kk) {
            double xv[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = wsm[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
    if (nslice == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
                if (t < a.T && e < a.E) a.logits[(int64_t)t * a.E + e] = (float)acc[i][j];
            }
        pdl_wait();
        return;
    }
    const int64_t TE = (int64_t)a.T * a.E;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
            if (t < a.T && e < a.E) part[sl * TE + (int64_t)t * a.E + e] = acc[i][j];
        }
    __threadfence();
    __syncthreads();
    const int tile = blockIdx.y * gridDim.x + blockIdx.x;
    if (tid == 0) {
        const int done = atomicAdd(tilecnt + tile, 1);
        last = done == nslice - 1;
        if (last) tilecnt[tile] = 0;             // ready for the next call
    }
    __syncthreads();
    if (last) {
        __threadfence();
        // slice by slice for all 16 of the thread's outputs at once (16
        // independent loads per slice in flight), each output still summed in
        // slice order
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
#pragma unroll 2
        for (int q = 0; q < nslice; ++q) {
            const double *pq = part + q * TE;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
                    if (t < a.T && e < a.E) acc[i][j] += __ldcg(pq + (int64_t)t * a.E + e);
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + ty + 16 * i, e = e0 + tx + 16 * j;
                if (t < a.T && e < a.E) a.logits[(int64_t)t * a.E + e] = (float)acc[i][j];
            }
    }
    pdl_wait();
}

// Slices for the split kernel: about two CTAs per SM, K slices of whole chunks.
inline int router_slices(int T, int E, int H)
{
    const int tiles = ((E + RS_E - 1) / RS_E) * ((T + RS_T - 1) / RS_T);
    int s = 1;
    while (tiles * s * 2 <= 2 * 148 && (H / RS_KC) % (s * 2) == 0 && s * 2 <= 64) s *= 2;
    return s;
}

// One warp per token.  Dynamic shared memory per warp: s[E], sc[E] (f32),
// gscore[G] (f32), kept[G] (int), sel[32] (int, the chosen experts in order).
__host__ __device__ inline size_t select_smem_per_warp(int E, int G) { return (size_t)(2 * E + 2 * G + 32) * 4; }

// The selection of token t by one warp; wsm: select_smem_per_warp(E, G) bytes
// of shared memory of its own.
__device__ __forceinline__ void select_token_warp(const RouterArgs &a, int t, int lane, unsigned char *wsm)
{
    const int E = a.E, G = a.G, gs = a.E / a.G;
    float *s_s = reinterpret_cast<float *>(wsm);
    float *sc_s = s_s + E;
    float *gsc = sc_s + E;
    int *kept = reinterpret_cast<int *>(gsc + G);
    int *sel = kept + G;

    for (int e = lane; e < E; e += 32) {
        const float lg = a.logits[(int64_t)t * E + e];
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
    // candidates of this lane: experts lane + 32 i in kept groups
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
        if (lane == 0) sel[j] = be;
    }
    __syncwarp();
    // weights: s_j / sum(s) * rsf, the sum in double in selection order
    double ssum = 0.0;
    if (lane == 0)
        for (int j = 0; j < a.k; ++j) ssum += (double)s_s[sel[j]];
    ssum = __shfl_sync(0xffffffffu, ssum, 0);
    const int e = lane < a.k ? sel[lane] : 0;
    const float wv = lane < a.k ? (float)((double)s_s[e] / ssum * (double)a.rsf) : 0.f;
    // adaptive top-p (when on): dropped slots become idx = -1, w = 0
    const bool keep = a.topp_thr > 0.0 ? warp_topp_keep(lane, a.k, wv, a.topp_thr) : true;
    if (lane < a.k) {
        a.idx[(int64_t)t * a.k + lane] = keep ? e : -1;
        a.w[(int64_t)t * a.k + lane] = keep ? wv : 0.f;
    }
}

// The same selection with every value in registers, for E a multiple of 32
// (at most 32 * NE) and groups of a multiple of 32 experts: lane l holds
// experts l + 32 i.  Group top-2 sums come from a butterfly over (top1, top2)
// pairs, all groups at once; the kept groups are ranked in registers; the k
// picks are warp arg-max rounds (ties to the lower expert); the weight sum is
// taken in double in pick order.  Same results as select_token_warp.
template <int NE>
__device__ __forceinline__ void select_token_warp_reg(const RouterArgs &a, int t, int lane)
{
    const int E = a.E, G = a.G, gs = E / G, ne = E / 32, gi = gs / 32;   // gi: i's per group
    float s[NE], sc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) {
        s[i] = 0.f;
        sc[i] = -INFINITY;
        if (i < ne) {
            const int e = lane + 32 * i;
            const float lg = a.logits[(int64_t)t * E + e];
            s[i] = (float)(1.0 / (1.0 + exp(-(double)lg)));
            sc[i] = __fadd_rn(s[i], a.bias[e]);
        }
    }
    // group scores: group g holds i in [g*gi, (g+1)*gi) of every lane
    float gsc[NE];
#pragma unroll
    for (int g = 0; g < NE; ++g) {
        float t1 = -INFINITY, t2 = -INFINITY;
        if (g < G) {
#pragma unroll
            for (int i = 0; i < NE; ++i)
                if (i >= g * gi && i < (g + 1) * gi) {
                    const float v = sc[i];
                    if (v > t1) { t2 = t1; t1 = v; }
                    else if (v > t2) { t2 = v; }
                }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float b1 = __shfl_xor_sync(0xffffffffu, t1, o), b2 = __shfl_xor_sync(0xffffffffu, t2, o);
            const float hi = fmaxf(t1, b1), lo = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
            t1 = hi;
            t2 = lo;
        }
        gsc[g] = gs >= 2 ? __fadd_rn(t1, t2) : t1;
    }
    // kept groups: rank among the G scores (ties to the lower group)
    uint32_t kept = 0;
#pragma unroll
    for (int g = 0; g < NE; ++g) {
        if (g >= G) continue;
        int rank = 0;
#pragma unroll
        for (int h = 0; h < NE; ++h)
            if (h < G) rank += (gsc[h] > gsc[g]) || (gsc[h] == gsc[g] && h < g);
        if (rank < a.Gk) kept |= 1u << g;
    }
    uint32_t avail = 0;       // bit i: expert lane + 32 i is a candidate not yet taken
#pragma unroll
    for (int i = 0; i < NE; ++i)
        if (i < ne && (kept >> (i / gi) & 1u)) avail |= 1u << i;
    int my_e = 0;
    float my_w = 0.f;
    double ssum = 0.0;
    for (int j = 0; j < a.k; ++j) {
        float best = -INFINITY;
        int be = 0x7fffffff, bi = -1;
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (avail >> i & 1u) {
                const int e = lane + 32 * i;
                if (be == 0x7fffffff || sc[i] > best) { best = sc[i]; be = e; bi = i; }
            }
        float bs = 0.f;       // the unbiased score of this lane's best candidate
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (i == bi) bs = s[i];
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float os = __shfl_xor_sync(0xffffffffu, bs, o);
            const bool better = (oe != 0x7fffffff) && (be == 0x7fffffff || ob > best || (ob == best && oe < be));
            if (better) { best = ob; be = oe; bs = os; }
        }
        if (be == 0x7fffffff) {      // cannot happen for a validated configuration
            if (lane == 0) raise_status(DERR_BOUNDS);
            return;
        }
        if ((be & 31) == lane) avail &= ~(1u << (be >> 5));
        ssum += (double)bs;
        if (lane == j) {
            my_e = be;
            my_w = bs;
        }
    }
    const float wv = lane < a.k ? (float)((double)my_w / ssum * (double)a.rsf) : 0.f;
    const bool keep = a.topp_thr > 0.0 ? warp_topp_keep(lane, a.k, wv, a.topp_thr) : true;
    if (lane < a.k) {
        a.idx[(int64_t)t * a.k + lane] = keep ? my_e : -1;
        a.w[(int64_t)t * a.k + lane] = keep ? wv : 0.f;
    }
}

// Whether select_token_warp_reg<8> takes this configuration.
__host__ __device__ inline bool select_reg_ok(int E, int G)
{
    return E % 32 == 0 && E <= 256 && G > 0 && E % G == 0 && (E / G) % 32 == 0;
}

__global__ void __launch_bounds__(256) k_router_select(RouterArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + wid;
    pdl_wait();
    pdl_trigger();
    if (t >= a.T) return;
    if (select_reg_ok(a.E, a.G)) select_token_warp_reg<8>(a, t, lane);
    else select_token_warp(a, t, lane, smem_raw + select_smem_per_warp(a.E, a.G) * wid);
}

// Selection and batch-union permutation of a small batch in one CTA of 1024
// threads: warp t selects token t's experts (written to a.idx / a.w), then the
// whole CTA sorts the assignments.  Saves a launch on the decode path.
__global__ void __launch_bounds__(1024, 1) k_select_permute(RouterArgs a, qrx_perm p, uint64_t *__restrict__ usage)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    if (wid < a.T) {
        if (select_reg_ok(a.E, a.G)) select_token_warp_reg<8>(a, wid, lane);
        else select_token_warp(a, wid, lane, smem_raw + select_smem_per_warp(a.E, a.G) * wid);
    }
    __syncthreads();        // the selection (global a.idx) is visible to the whole CTA
    permute_cta(a.idx, a.T * a.k, a.E, p, usage, reinterpret_cast<int *>(smem_raw));
}

bool select_permute_fused_ok(int T, int E, int G)
{
    return T <= 32 && T * select_smem_per_warp(E, G) <= 200 * 1024 && permute_smem_bytes(E) <= 200 * 1024;
}

cudaError_t launch_select_permute(const RouterArgs &a, const qrx_perm &p, uint64_t *usage, cudaStream_t st)
{
    const size_t smem = std::max((size_t)a.T * select_smem_per_warp(a.E, a.G), permute_smem_bytes(a.E));
    if (smem > 48 * 1024) {
        const cudaError_t err =
            cudaFuncSetAttribute(k_select_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    return launch_k(k_select_permute, dim3(1), dim3(1024), smem, st, a, p, usage);
}

// Adaptive expert top-p on a router output already in memory: warp per token.
__global__ void __launch_bounds__(256) k_topp_prune(int32_t *__restrict__ idx, float *__restrict__ w, int T,
                                                    int k, double thr)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    pdl_wait();
    pdl_trigger();
    if (t >= T) return;
    const int64_t a = (int64_t)t * k + lane;
    const float wv = lane < k ? w[a] : 0.f;
    const int32_t e = lane < k ? idx[a] : -1;
    const bool keep = warp_topp_keep(lane, k, wv, thr);
    if (lane < k) {
        idx[a] = keep ? e : -1;
        w[a] = keep ? wv : 0.f;
    }
}

cudaError_t launch_topp_prune(int32_t *idx, float *w, int T, int k, double thr, cudaStream_t st)
{
    return launch_k(k_topp_prune, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, st, idx, w, T, k, thr);
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t st, bool select)
{
    cudaError_t err;
    if (a.T <= RG_TSPLIT && a.H <= 16 * 32 * RG_W4) {
        const unsigned grid = (unsigned)((a.E + RG_ROWS - 1) / RG_ROWS);
        err = launch_k(a.x_bf16 ? k_router_gemv<true> : k_router_gemv<false>, dim3(grid), dim3(256), 0,
                       st, a);
    } else if (a.part && a.tilecnt && a.H % RS_KC == 0) {
        const int ns = router_slices(a.T, a.E, a.H);
        dim3 grid((a.E + RS_E - 1) / RS_E, (a.T + RS_T - 1) / RS_T, ns);
        if (ns > 1) {                            // the tile counters start at zero (the workspace is not cleared)
            err = cudaMemsetAsync(a.tilecnt, 0, sizeof(int) * grid.x * grid.y, st);
            if (err != cudaSuccess) return err;
        }
        err = launch_k(a.x_bf16 ? k_router_split<true> : k_router_split<false>, grid, dim3(256), 0, st, a, ns,
                       a.part, a.tilecnt);
    } else {
        dim3 grid((a.E + RT_E - 1) / RT_E, (a.T + RT_T - 1) / RT_T);
        err = launch_k(a.x_bf16 ? k_router_tile<true> : k_router_tile<false>, grid, dim3(256), 0, st, a);
    }
    if (err != cudaSuccess || !select) return err;
    const size_t smem = (size_t)8 * select_smem_per_warp(a.E, a.G);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(k_router_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return err;
    }
    return launch_k(k_router_select, dim3((a.T + 7) / 8), dim3(256), smem, st, a);
}

}  // namespace qrx
