// k_ffn_gemv.cuh -- expert FFN over the batch union, GEMV-shaped (few tokens
// per expert): HBM-bound streaming of packed weights with integer dots.
//
// README "JustVugg/colibri", section "已实现的功能": batch-union MoE (each
// unique expert of a batch read once and applied to all positions routed to
// it), int8 / packed int4 / packed int2 weights with per-row scales
// dequantised on use, Q8_0-style int8-activation integer dot kernels.  The
// expert is a SwiGLU FFN: h = silu(s_g Q_g x) * (s_u Q_u x), y = s_d Q_d h.
//
// Work decomposition.  A "slot" is one expert of the union (or the shared
// expert) with the list of token positions routed to it, cut into token
// groups of at most TS tokens.  Each slot's matrix is cut into blocks of RB
// rows; the (slot, group, block) units are split into contiguous ranges of
// equal estimated cost (weight streaming plus per-token dot work), one range
// per CTA (one CTA per SM).  Inside a CTA, a "team" of CPR threads covers
// one row (thread c loads 16-byte chunk c of the row), and each team handles R
// consecutive rows of a block.  The slot's activations are staged once into
// shared memory as digit planes (see qrx_dev.cuh) for up to TS tokens; each
// thread keeps its R weight chunks in registers and runs every staged token
// over them, so a weight byte is read from HBM once per slot.  For gate/up
// the matrix rows are interleaved (gate row i, up row i) so the SwiGLU is
// applied where both rows' sums meet.  Reductions are fixed-order (warp
// butterflies, then warp partials in index order): results are deterministic.
#pragma once
#include "qrx_dev.cuh"

namespace qrx {

constexpr int GV_NT = 384;   // threads per CTA (12 warps)
constexpr int GV_R = 8;      // rows per team per block

struct GemvP {
    int K, rows, row_bytes, cpr, tpc, rb, nblk, ts, wpt, redn;
    const uint8_t *w;
    int64_t w_stride;        // bytes between experts' matrices
    const float *s;
    int64_t s_stride;        // floats between experts' scale vectors
    const uint8_t *w_sh;
    const float *s_sh;
    int routed, shared;
    const int32_t *offsets, *sorted, *union_ids, *n_union;
    int E, k, T;
    int afmt;
    const void *x;           // gate/up input rows (token index)
    const int8_t *xq;
    const float *xd;
    const float *hin;        // down input rows
    int64_t hin_ld, sh_in_row0;
    float *out;
    int64_t out_ld, sh_out_row0;
};

template <int N>
__device__ __forceinline__ void tr_step(float *v, int lane, int off)
{
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        const float send = up ? v[i] : v[i + N / 2];
        const float keep = up ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
}

// Transposed butterfly: V values per lane -> lane holds the warp total of value
// index lane >> (5 - log2 V).
template <int V>
__device__ __forceinline__ float warp_tr_reduce(float (&v)[V], int lane)
{
    int off = 16;
    if constexpr (V >= 32) { tr_step<32>(v, lane, off); off >>= 1; }
    if constexpr (V >= 16) { tr_step<16>(v, lane, off); off >>= 1; }
    if constexpr (V >= 8) { tr_step<8>(v, lane, off); off >>= 1; }
    if constexpr (V >= 4) { tr_step<4>(v, lane, off); off >>= 1; }
    if constexpr (V >= 2) { tr_step<2>(v, lane, off); off >>= 1; }
    for (; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    return v[0];
}

template <int V> struct Log2 { static constexpr int value = 1 + Log2<V / 2>::value; };
template <> struct Log2<1> { static constexpr int value = 0; };

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int WB, int NDIG, int TP, bool GATEUP>
__global__ void __launch_bounds__(GV_NT, 1) k_ffn_gemv(const GemvP p)
{
    using F = Fmt<WB>;
    constexpr int R = GV_R, V = R * TP, LV = Log2<V>::value;
    constexpr int NBC = WB == 2 ? 2 : 1;              // scale blocks touched by a chunk
    extern __shared__ __align__(16) unsigned char smem[];
    const int K = p.K, nb = K / 32, cpr = p.cpr;
    uint32_t *dig = reinterpret_cast<uint32_t *>(smem);
    float *bsc = reinterpret_cast<float *>(smem + (size_t)p.ts * NDIG * K);
    float *red = bsc + (size_t)p.ts * nb;
    int *tin = reinterpret_cast<int *>(red + 2 * p.redn);
    int *tout = tin + p.ts;
    int64_t *pre = reinterpret_cast<int64_t *>(tout + p.ts);   // [nslots + 1], 8-aligned

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid % cpr, team = tid / cpr, wit = c >> 5;

    // ---- cost-weighted partition of (slot, token group, row block) work units.
    // A unit costs BWU (streaming its weights) + its token count (dot work);
    // slot s has ceil(ntok/TS) groups, all full but the last, so its cost is
    // nblk * (BWU * groups + ntok).  pre[] holds the prefix over slots; each
    // CTA owns the units whose cost start falls in its equal share.
    constexpr int64_t BWU = NDIG == 1 ? 8 : 3;
    const int nu = p.routed ? *p.n_union : 0;
    const int nslots = nu + (p.shared ? 1 : 0);
    if (tid < 32) {
        int64_t run = 0;
        for (int s0 = 0; s0 < nslots; s0 += 32) {
            const int s = s0 + lane;
            int64_t cost = 0;
            if (s < nslots) {
                int ntok = p.T;
                if (s < nu) {
                    const int e = p.union_ids[s];
                    ntok = (e >= 0 && e < p.E) ? p.offsets[e + 1] - p.offsets[e] : 0;
                }
                const int groups = (ntok + p.ts - 1) / p.ts;
                cost = (int64_t)p.nblk * (BWU * groups + ntok);
            }
            int64_t inc = cost;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            if (s < nslots) pre[s] = run + inc - cost;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pre[nslots] = run;
    }
    __syncthreads();
    const int64_t Ctot = pre[nslots];
    const int64_t c0 = Ctot * blockIdx.x / gridDim.x, c1 = Ctot * (blockIdx.x + 1) / gridDim.x;
    int sfirst = 0;
    {   // last slot whose prefix is <= c0
        int lo = 0, hi = nslots;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= c0) lo = mid; else hi = mid;
        }
        sfirst = lo;
    }
    int pass = 0;

    for (int s = sfirst; s < nslots && pre[s] < c1; ++s) {
        int p0, ntok;
        const uint8_t *W;
        const float *S;
        const bool is_routed = s < nu;
        if (is_routed) {
            const int e = p.union_ids[s];
            if (e < 0 || e >= p.E) { if (tid == 0) raise_status(DERR_BADIDX); return; }
            p0 = p.offsets[e];
            ntok = p.offsets[e + 1] - p0;
            W = p.w + (int64_t)e * p.w_stride;
            S = p.s + (int64_t)e * p.s_stride;
        } else {
            p0 = 0;
            ntok = p.T;
            W = p.w_sh;
            S = p.s_sh;
        }
        for (int tg = 0, j = 0; tg < ntok; tg += p.ts, ++j) {
            const int nt = min(p.ts, ntok - tg);
            const int64_t gstart = pre[s] + (int64_t)p.nblk * j * (BWU + p.ts);
            const int64_t cb = BWU + nt;
            int64_t bfirst = c0 > gstart ? (c0 - gstart + cb - 1) / cb : 0;
            int64_t bend = c1 > gstart ? (c1 - gstart + cb - 1) / cb : 0;
            if (bend > p.nblk) bend = p.nblk;
            if (bfirst >= bend) continue;
            __syncthreads();                       // previous group's readers are done
            if (tid < nt) {
                const int i = tg + tid;
                if (is_routed) {
                    const int pos = p0 + i;
                    tin[tid] = GATEUP ? p.sorted[pos] / p.k : pos;
                    tout[tid] = pos;
                } else {
                    tin[tid] = GATEUP ? i : (int)p.sh_in_row0 + i;
                    tout[tid] = (int)p.sh_out_row0 + i;
                }
            }
            __syncthreads();
            // ---- stage the tokens' activations as digit planes
            unsigned char *digb = reinterpret_cast<unsigned char *>(dig);
            for (int blk = warp; blk < nt * nb; blk += GV_NT / 32) {
                const int i = blk / nb, bb = blk % nb;
                const int elem = bb * 32 + lane;
                const int64_t row = tin[i];
                int8_t d[3] = {0, 0, 0};
                float sig = 0.f;
                if constexpr (NDIG == 1) {
                    if constexpr (GATEUP) {
                        d[0] = p.xq[row * K + elem];
                        sig = p.xd[row * nb + bb];
                    } else {
                        const float v = p.hin[row * p.hin_ld + elem];
                        const float amax = warp_max(fabsf(v));
                        if (amax != 0.f) {
                            d[0] = (int8_t)q8_code(v, __fdiv_rn(127.f, amax));
                            sig = __fdiv_rn(amax, 127.f);
                        }
                    }
                } else {
                    float v;
                    if constexpr (GATEUP) {
                        if (p.afmt == QRX_A_BF16)
                            v = __bfloat162float(
                                reinterpret_cast<const __nv_bfloat16 *>(p.x)[row * K + elem]);
                        else
                            v = reinterpret_cast<const float *>(p.x)[row * K + elem];
                    } else {
                        v = p.hin[row * p.hin_ld + elem];
                        if (p.afmt == QRX_A_BF16) v = __bfloat162float(__float2bfloat16_rn(v));
                    }
                    const float amax = warp_max(fabsf(v));
                    if (amax != 0.f) {
                        const int sh = fixed_shift(amax);
                        split3(__float2int_rn(ldexpf(v, sh)), d[0], d[1], d[2]);
                        sig = ldexpf(1.f, -sh);
                    }
                }
                const int cc = elem / F::EPC, l = elem % F::EPC;
                int wd, by;
                digit_slot<WB>(l, wd, by);
#pragma unroll
                for (int pl = 0; pl < NDIG; ++pl)
                    digb[((((size_t)i * NDIG + pl) * cpr + cc) * F::DW + wd) * 4 + by] =
                        (unsigned char)d[pl];
                if (lane == 0) bsc[i * nb + bb] = sig;
            }
            __syncthreads();

            // ---- this group's blocks in my range
            for (int64_t bb = bfirst; bb < bend; ++bb) {
                const int rblk = (int)bb;
                const int rowbase = rblk * p.rb + team * R;
                uint4 wv[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int row = rowbase + r;
                    wv[r] = row < p.rows
                                ? ld_stream16(W + (int64_t)row * p.row_bytes + (int64_t)c * 16)
                                : make_uint4(0u, 0u, 0u, 0u);
                }
                for (int t0 = 0; t0 < nt; t0 += TP) {
                    float part[V];
#pragma unroll
                    for (int tt = 0; tt < TP; ++tt) {
                        if (t0 + tt < nt) {
                            const int ti = t0 + tt;
                            uint32_t dw[NDIG][F::DW];
#pragma unroll
                            for (int pl = 0; pl < NDIG; ++pl) {
                                const uint4 *src = reinterpret_cast<const uint4 *>(
                                    dig + (((size_t)ti * NDIG + pl) * cpr + c) * F::DW);
#pragma unroll
                                for (int q4 = 0; q4 < F::DW / 4; ++q4) {
                                    const uint4 v4 = src[q4];
                                    dw[pl][4 * q4 + 0] = v4.x;
                                    dw[pl][4 * q4 + 1] = v4.y;
                                    dw[pl][4 * q4 + 2] = v4.z;
                                    dw[pl][4 * q4 + 3] = v4.w;
                                }
                            }
                            float sig[NBC];
                            int corr[NBC][NDIG];
#pragma unroll
                            for (int bc = 0; bc < NBC; ++bc) {
                                const int sb = WB == 8 ? (c >> 1) : (WB == 4 ? c : 2 * c + bc);
                                sig[bc] = bsc[ti * nb + sb];
#pragma unroll
                                for (int pl = 0; pl < NDIG; ++pl) {
                                    int sum = 0;
                                    if constexpr (F::OFF != 0) {
                                        constexpr int WPB = F::DW / NBC;
#pragma unroll
                                        for (int q = 0; q < WPB; ++q)
                                            sum = dp4a(dw[pl][bc * WPB + q], 0x01010101u, sum);
                                    }
                                    corr[bc][pl] = -F::OFF * sum;
                                }
                            }
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                int acc[NBC][NDIG];
#pragma unroll
                                for (int bc = 0; bc < NBC; ++bc)
#pragma unroll
                                    for (int pl = 0; pl < NDIG; ++pl) acc[bc][pl] = corr[bc][pl];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    uint32_t u[F::UPW];
                                    unpack_word<WB>(word_of(wv[r], i), u);
                                    const int bc = WB == 2 ? (i >> 1) : 0;
#pragma unroll
                                    for (int j = 0; j < F::UPW; ++j)
#pragma unroll
                                        for (int pl = 0; pl < NDIG; ++pl)
                                            acc[bc][pl] = dp4a(u[j], dw[pl][i * F::UPW + j], acc[bc][pl]);
                                }
                                float v = 0.f;
#pragma unroll
                                for (int bc = 0; bc < NBC; ++bc) {
                                    float cv;
                                    if constexpr (NDIG == 3)
                                        cv = fmaf(__int2float_rn(acc[bc][2]), 65536.f,
                                                  __int2float_rn(acc[bc][0] + 256 * acc[bc][1]));
                                    else
                                        cv = __int2float_rn(acc[bc][0]);
                                    v = fmaf(sig[bc], cv, v);
                                }
                                part[r * TP + tt] = v;
                            }
                        } else {
#pragma unroll
                            for (int r = 0; r < R; ++r) part[r * TP + tt] = 0.f;
                        }
                    }
                    // ---- reduce over the team
                    float *rbuf = red + (pass & 1) * p.redn;
                    if (cpr >= 32) {
                        const float tot = warp_tr_reduce<V>(part, lane);
                        if ((lane & ((1 << (5 - LV)) - 1)) == 0)
                            rbuf[(team * p.wpt + wit) * V + (lane >> (5 - LV))] = tot;
                    } else {
#pragma unroll
                        for (int vi = 0; vi < V; ++vi) {
                            float xv = part[vi];
                            for (int o = cpr >> 1; o; o >>= 1) xv += __shfl_xor_sync(0xffffffffu, xv, o);
                            if (c == 0) rbuf[team * V + vi] = xv;
                        }
                    }
                    __syncthreads();
                    // ---- finalize: scales, SwiGLU, store
                    if constexpr (GATEUP) {
                        const int per_team = (R / 2) * TP;
                        for (int f = tid; f < p.tpc * per_team; f += GV_NT) {
                            const int tf = f / per_team, rem = f % per_team;
                            const int q = rem / TP, tt = rem % TP;
                            const int row_g = rblk * p.rb + tf * R + 2 * q;
                            if (t0 + tt >= nt || row_g >= p.rows) continue;
                            float G = 0.f, U = 0.f;
                            for (int w2 = 0; w2 < p.wpt; ++w2) {
                                G += rbuf[(tf * p.wpt + w2) * V + (2 * q) * TP + tt];
                                U += rbuf[(tf * p.wpt + w2) * V + (2 * q + 1) * TP + tt];
                            }
                            const float g = S[row_g] * G, u = S[row_g + 1] * U;
                            p.out[(int64_t)tout[t0 + tt] * p.out_ld + (row_g >> 1)] = silu_mul(g, u);
                        }
                    } else {
                        const int per_team = R * TP;
                        for (int f = tid; f < p.tpc * per_team; f += GV_NT) {
                            const int tf = f / per_team, rem = f % per_team;
                            const int r = rem / TP, tt = rem % TP;
                            const int row = rblk * p.rb + tf * R + r;
                            if (t0 + tt >= nt || row >= p.rows) continue;
                            float Y = 0.f;
                            for (int w2 = 0; w2 < p.wpt; ++w2) Y += rbuf[(tf * p.wpt + w2) * V + r * TP + tt];
                            p.out[(int64_t)tout[t0 + tt] * p.out_ld + row] = S[row] * Y;
                        }
                    }
                    ++pass;
                }
            }
        }
    }
}

// ---------------------------------------------------------------- host side
struct GemvPlan {
    GemvP p;
    size_t smem;
    int tp;
};

static inline int gemv_smem_limit() { return 200 * 1024; }

// Fill geometry for a matrix of `rows` x `K` codes at `wbits`, for slots of
// at most `maxtok` tokens with NDIG digit planes.
static inline bool gemv_plan(GemvPlan &pl, int wbits, int ndig, int K, int rows, int maxtok,
                             int maxslots)
{
    GemvP &p = pl.p;
    p.K = K;
    p.rows = rows;
    p.row_bytes = K * wbits / 8;
    p.cpr = p.row_bytes / 16;
    if (p.cpr <= 0 || GV_NT % p.cpr != 0) return false;
    if (p.cpr < 32 && (32 % p.cpr) != 0) return false;
    if (p.cpr > 32 && (p.cpr % 32) != 0) return false;
    p.tpc = GV_NT / p.cpr;
    p.rb = p.tpc * GV_R;
    p.nblk = (rows + p.rb - 1) / p.rb;
    p.wpt = p.cpr >= 32 ? p.cpr / 32 : 1;
    pl.tp = maxtok <= 1 ? 1 : (ndig == 1 ? 4 : 2);
    const int V = GV_R * pl.tp;
    p.redn = p.tpc * p.wpt * V;
    const size_t fixed = (size_t)2 * p.redn * 4 + 64 + (size_t)8 * (maxslots + 2);
    const size_t per_tok = (size_t)ndig * K + (size_t)(K / 32) * 4 + 8;
    const size_t lim = (size_t)gemv_smem_limit();
    if (fixed + per_tok > lim) return false;
    int ts = (int)((lim - fixed) / per_tok);
    if (ts > maxtok) ts = maxtok;
    if (ts < 1) ts = 1;
    p.ts = ts;
    pl.smem = (size_t)ts * ndig * K + (size_t)ts * (K / 32) * 4 + (size_t)2 * p.redn * 4 +
              (size_t)2 * (ts + 1) * 4 + (size_t)8 * (maxslots + 2);
    return true;
}

template <int WB, int NDIG, int TP, bool GU>
static cudaError_t gemv_go(const GemvPlan &pl, int grid, cudaStream_t st)
{
    auto kern = k_ffn_gemv<WB, NDIG, TP, GU>;
    static unsigned long long configured = 0;   // bit per device: max dynamic smem set
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   gemv_smem_limit() + 4096);
        if (err != cudaSuccess) return err;
        if (dev < 64) configured |= 1ull << dev;
    }
    kern<<<grid, GV_NT, pl.smem, st>>>(pl.p);
    return cudaGetLastError();
}

template <bool GU>
static cudaError_t gemv_dispatch(const GemvPlan &pl, int wbits, int ndig, int grid, cudaStream_t st)
{
#define QRX_GV(WB, ND, TP) \
    if (wbits == WB && ndig == ND && pl.tp == TP) return gemv_go<WB, ND, TP, GU>(pl, grid, st);
    QRX_GV(4, 3, 1) QRX_GV(4, 3, 2) QRX_GV(4, 1, 1) QRX_GV(4, 1, 4)
    QRX_GV(8, 3, 1) QRX_GV(8, 3, 2) QRX_GV(8, 1, 1) QRX_GV(8, 1, 4)
    QRX_GV(2, 3, 1) QRX_GV(2, 3, 2) QRX_GV(2, 1, 1) QRX_GV(2, 1, 4)
#undef QRX_GV
    return cudaErrorInvalidValue;
}

static inline void gemv_common(GemvP &p, const FfnArgs &a)
{
    p.routed = a.routed;
    p.shared = a.shared;
    p.offsets = a.offsets;
    p.sorted = a.sorted;
    p.union_ids = a.union_ids;
    p.n_union = a.n_union;
    p.E = a.E;
    p.k = a.k;
    p.T = a.T;
    p.afmt = a.afmt;
    p.x = a.x;
    p.xq = a.xq;
    p.xd = a.xd;
}

cudaError_t launch_ffn_gateup(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    GemvPlan pl;
    if (!gemv_plan(pl, a.wbits, ndig, a.H, 2 * a.I, a.T, a.E + 1)) return cudaErrorInvalidValue;
    GemvP &p = pl.p;
    gemv_common(p, a);
    p.w = a.w13;
    p.w_stride = (int64_t)2 * a.I * p.row_bytes;
    p.s = a.s13;
    p.s_stride = (int64_t)2 * a.I;
    p.w_sh = a.w13_sh;
    p.s_sh = a.s13_sh;
    p.hin = nullptr;
    p.hin_ld = 0;
    p.sh_in_row0 = 0;
    p.out = a.h;
    p.out_ld = a.h_ld;
    p.sh_out_row0 = a.sh_h_row0;
    return gemv_dispatch<true>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_ffn_down(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    GemvPlan pl;
    if (!gemv_plan(pl, a.wbits, ndig, a.I, a.H, a.T, a.E + 1)) return cudaErrorInvalidValue;
    GemvP &p = pl.p;
    gemv_common(p, a);
    p.w = a.w2;
    p.w_stride = (int64_t)a.H * p.row_bytes;
    p.s = a.s2;
    p.s_stride = a.H;
    p.w_sh = a.w2_sh;
    p.s_sh = a.s2_sh;
    p.hin = a.h;
    p.hin_ld = a.h_ld;
    p.sh_in_row0 = a.sh_h_row0;
    p.out = a.y;
    p.out_ld = a.y_ld;
    p.sh_out_row0 = a.sh_y_row0;
    return gemv_dispatch<false>(pl, a.wbits, ndig, num_sms, st);
}

}  // namespace qrx
